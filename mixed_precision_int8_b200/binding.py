"""ctypes binding of libllmint8.so (the C ABI in include/llmint8.h).

Argument marshalling only: every step of the layer runs in the library's
CUDA kernels. PyTorch provides device memory and streams. The functions keep
the C names; tensors are passed as device pointers, the stream as the current
torch stream. If the library is missing, loading fails loudly: there is no
CPU fallback.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libllmint8.so")

OK = 0
STATUS_NAMES = {0: "OK", -1: "ERR_NULL", -2: "ERR_SHAPE", -3: "ERR_ALIGN",
                -4: "ERR_WORKSPACE", -5: "ERR_CUDA", -6: "ERR_DEVICE_STATUS",
                -7: "ERR_ARG", -8: "ERR_UNSUPPORTED", -9: "ERR_TOO_LARGE"}
NOALLOC_MAX_SCRATCH_BYTES = 64 << 20  # LLMINT8_NOALLOC_MAX_SCRATCH_BYTES
# device status bits (LLMINT8_DEV_*)
DEV_TIMEOUT_SELFTEST = 0x20
DEV_OUTLIER_CAP = 0x40
SCALE_VECTORWISE = 0  # LLMINT8_SCALE_VECTORWISE: per row of X / column of W
# where the prefill path builds the fp16 outlier rows of W (LLMINT8_WO_*)
WO_SHARED, WO_BEFORE_GEMM, WO_EACH_CTA = 0, 1, 2
SCALE_TENSORWISE = 1  # LLMINT8_SCALE_TENSORWISE: one constant per tensor
# llmint8_matmul_opts.path (LLMINT8_PATH_*)
PATH_AUTO, PATH_PREFILL, PATH_DECODE, PATH_PREFILL_SINGLE, PATH_PREFILL_PAIR = 0, 1, 2, 3, 4

_c_i64, _c_i32, _c_f32 = ctypes.c_int64, ctypes.c_int32, ctypes.c_float
_vp, _sz = ctypes.c_void_p, ctypes.c_size_t


class llmint8_weight(ctypes.Structure):
    _fields_ = [("h", _c_i64), ("o", _c_i64), ("wq_dev", _vp), ("aw_dev", _vp),
                ("w16_dev", _vp)]


class llmint8_matmul_opts(ctypes.Structure):
    _fields_ = [("gemm_event_start", _vp), ("gemm_event_stop", _vp),
                ("ci_dev", _vp), ("path", _c_i32), ("launches", _c_i32),
                ("x_scale", _c_i32), ("max_outliers", _c_i32),
                ("status_host", _vp), ("wo_build", _c_i32)]


class Llmint8Error(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = code
        super().__init__(f"{fn} failed: {STATUS_NAMES.get(code, code)}"
                         f" ({status_string(code) if _lib is not None else ''})")


_lib = None


def load_library():
    """Load libllmint8.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} not found: build it with `python -m "
            "mixed_precision_int8_b200.build` (or __graft_entry__.build())")
    lib = ctypes.CDLL(LIB_PATH)
    sig = {
        "llmint8_status_string": ([_c_i32], ctypes.c_char_p),
        "llmint8_workspace_size": ([_c_i64, _c_i64, _c_i64], _sz),
        "llmint8_workspace_size_ex": ([_c_i64, _c_i64, _c_i64, _c_i64], _sz),
        "llmint8_workspace_size_host": ([_c_i64, _c_i64, _c_i64], _sz),
        "llmint8_workspace_size_host_ex": ([_c_i64, _c_i64, _c_i64, _c_i64], _sz),
        "llmint8_workspace_init": ([_vp, _sz, _vp], _c_i32),
        "llmint8_prepare_weight": ([_vp, _c_i64, _c_i64,
                                    ctypes.POINTER(llmint8_weight), _vp], _c_i32),
        "llmint8_prepare_weight_ex": ([_vp, _c_i64, _c_i64, _c_i32,
                                       ctypes.POINTER(llmint8_weight), _vp], _c_i32),
        "llmint8_prepare_weight_cols": ([_vp, _c_i64, _c_i64, _c_i64, _c_i64, _c_i32,
                                         ctypes.POINTER(llmint8_weight), _vp], _c_i32),
        "llmint8_quantize_rows_scratch_size": ([_c_i64], _sz),
        "llmint8_quantize_rows_ex": ([_vp, _c_i64, _c_i64, _c_f32, _c_i32, _vp,
                                      _vp, _vp, _vp, _vp, _vp, _sz, _vp], _c_i32),
        "llmint8_quantize_rows": ([_vp, _c_i64, _c_i64, _c_f32, _vp, _vp, _vp,
                                   _vp, _vp, _vp, _sz, _vp], _c_i32),
        "llmint8_matmul": ([_vp, _c_i64, ctypes.POINTER(llmint8_weight), _c_f32,
                            _vp, _vp, _sz, _vp], _c_i32),
        "llmint8_matmul_ex": ([_vp, _c_i64, ctypes.POINTER(llmint8_weight),
                               _c_f32, _vp, _vp, _sz,
                               ctypes.POINTER(llmint8_matmul_opts), _vp], _c_i32),
        "llmint8_matmul_host": ([_vp, _c_i64, ctypes.POINTER(llmint8_weight),
                                 _c_f32, _vp, _vp, _sz, _vp], _c_i32),
        "llmint8_matmul_host_ex": ([_vp, _c_i64, ctypes.POINTER(llmint8_weight),
                                    _c_f32, _vp, _vp, _sz,
                                    ctypes.POINTER(llmint8_matmul_opts), _vp], _c_i32),
        "llmint8_read_outlier_tiles": ([_vp, _sz, _c_i64, _c_i64, _c_i64, _vp,
                                        _vp, _vp, _vp], _c_i32),
        "llmint8_read_outlier_tiles_ex": ([_vp, _sz, _c_i64, _c_i64, _c_i64,
                                           _c_i64, _vp, _vp, _vp, _vp], _c_i32),
        "llmint8_read_device_status": ([_vp, _sz, _vp, _vp], _c_i32),
        "llmint8_decode_max_rows": ([], _c_i64),
        "llmint8_prefill_kernel": ([_c_i64, _c_i64, _c_i64], _c_i32),
        "llmint8_matmul_noalloc": ([_vp, _c_i64, ctypes.POINTER(llmint8_weight),
                                    _c_f32, _vp, _vp], _c_i32),
        "llmint8_wait_selftest": ([_vp, _sz, ctypes.c_uint64, _vp], _c_i32),
        "llmint8_noalloc_read_device_status": ([_vp, _vp], _c_i32),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    _lib = lib
    return lib


EXPORTED = ("llmint8_status_string", "llmint8_workspace_size",
            "llmint8_workspace_size_host", "llmint8_workspace_init",
            "llmint8_prepare_weight", "llmint8_quantize_rows_scratch_size",
            "llmint8_quantize_rows", "llmint8_matmul", "llmint8_matmul_ex",
            "llmint8_matmul_host", "llmint8_read_outlier_tiles",
            "llmint8_read_device_status", "llmint8_decode_max_rows",
            "llmint8_matmul_noalloc", "llmint8_wait_selftest",
            "llmint8_prepare_weight_ex", "llmint8_quantize_rows_ex",
            "llmint8_matmul_host_ex", "llmint8_workspace_size_ex",
            "llmint8_workspace_size_host_ex", "llmint8_read_outlier_tiles_ex",
            "llmint8_noalloc_read_device_status", "llmint8_prepare_weight_cols",
            "llmint8_prefill_kernel")


def status_string(code: int) -> str:
    return load_library().llmint8_status_string(code).decode()


def _check(fn: str, code: int):
    if code != OK:
        raise Llmint8Error(fn, code)


def _stream(stream: Optional[torch.cuda.Stream] = None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _f16_dev(t: torch.Tensor, name: str):
    if t.dtype != torch.float16 or not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA float16 tensor")


class PreparedWeight:
    """Device buffers of a prepared weight: wq int8 [o,h], aw float32 [o],
    and optionally the fp16 weight itself (w16 [h,o], kept referenced here)
    whose outlier rows then serve as the fp16 outlier rows of W."""

    def __init__(self, wq: torch.Tensor, aw: torch.Tensor,
                 w16: Optional[torch.Tensor] = None):
        self.wq = wq
        self.aw = aw
        self.w16 = w16
        self.o, self.h = wq.shape
        self.c = llmint8_weight(self.h, self.o, wq.data_ptr(), aw.data_ptr(),
                                w16.data_ptr() if w16 is not None else None)


class Workspace:
    """A caller-owned device workspace (torch uint8 buffer) for one stream.

    max_outliers (0: h, any alpha) sizes its outlier tiles; calls on it pass
    the same capacity to the library."""

    def __init__(self, s: int, h: int, o: int, device=None, host: bool = False,
                 max_outliers: int = 0):
        lib = load_library()
        size_fn = (lib.llmint8_workspace_size_host_ex if host
                   else lib.llmint8_workspace_size_ex)
        self.nbytes = int(size_fn(s, h, o, int(max_outliers)))
        if self.nbytes == 0:
            raise ValueError(f"invalid workspace size arguments {(s, h, o, max_outliers)}")
        self.buf = torch.empty(self.nbytes, dtype=torch.uint8,
                               device=device or "cuda")
        self.s, self.h, self.o = s, h, o
        self.max_outliers = int(max_outliers)
        _check("llmint8_workspace_init",
               lib.llmint8_workspace_init(_ptr(self.buf), self.nbytes, _stream()))


def llmint8_workspace_size(s: int, h: int, o: int, max_outliers: int = 0) -> int:
    return int(load_library().llmint8_workspace_size_ex(s, h, o, int(max_outliers)))


class HostStatusWord:
    """A pinned host int32 that the device writes: passed as status_host, it
    receives the status bits of each call's kernels, and the next call on it
    raises ERR_DEVICE_STATUS (code -6) before enqueuing anything."""

    def __init__(self):
        self.t = torch.zeros((1,), dtype=torch.int32).pin_memory()

    @property
    def value(self) -> int:
        return int(self.t[0].item())

    def clear(self):
        self.t[0] = 0


def llmint8_decode_max_rows() -> int:
    return int(load_library().llmint8_decode_max_rows())


def llmint8_prefill_kernel(s: int, h: int, o: int) -> int:
    """PATH_* value of the kernel the automatic choice runs for [s,h] x [h,o]
    on the current device (PATH_DECODE, PATH_PREFILL_SINGLE or
    PATH_PREFILL_PAIR)."""
    r = int(load_library().llmint8_prefill_kernel(int(s), int(h), int(o)))
    _check("llmint8_prefill_kernel", r if r < 0 else 0)
    return r


def llmint8_prepare_weight(W: torch.Tensor, stream=None,
                           keep_fp16: bool = False,
                           w_scale: int = SCALE_VECTORWISE) -> PreparedWeight:
    """W fp16 [h,o] on the GPU -> PreparedWeight (int8 [o,h] codes + scales).

    With keep_fp16 the weight keeps W (a reference, not a copy) and the
    layer's fp16 outlier rows of W are W's own values. w_scale =
    SCALE_TENSORWISE gives every column the one absmax of all of W."""
    _f16_dev(W, "W")
    h, o = W.shape
    wq = torch.empty((o, h), dtype=torch.int8, device=W.device)
    aw = torch.empty((o,), dtype=torch.float32, device=W.device)
    pw = PreparedWeight(wq, aw, W if keep_fp16 else None)
    _check("llmint8_prepare_weight_ex", load_library().llmint8_prepare_weight_ex(
        _ptr(W), h, o, int(w_scale), ctypes.byref(pw.c), _stream(stream)))
    return pw


def llmint8_prepare_weight_cols(W: torch.Tensor, col0: int, o: int, stream=None,
                                w_scale: int = SCALE_VECTORWISE) -> PreparedWeight:
    """Columns [col0, col0 + o) of W fp16 [h, o_total] (on the GPU) prepared
    as a weight of their own: one column-parallel shard."""
    _f16_dev(W, "W")
    h, ldw = W.shape
    wq = torch.empty((o, h), dtype=torch.int8, device=W.device)
    aw = torch.empty((o,), dtype=torch.float32, device=W.device)
    pw = PreparedWeight(wq, aw, None)
    _check("llmint8_prepare_weight_cols", load_library().llmint8_prepare_weight_cols(
        _ptr(W), h, ldw, int(col0), int(o), int(w_scale), ctypes.byref(pw.c),
        _stream(stream)))
    return pw


def llmint8_quantize_rows(X: torch.Tensor, alpha: float = 6.0, stream=None,
                          x_scale: int = SCALE_VECTORWISE):
    """Steps 1 and 4 (activation side) -> (Xq, ax, flags, idx, n_outliers).

    x_scale = SCALE_TENSORWISE quantises all rows against one constant.

    n_outliers is a 1-element device tensor (it is never read back here);
    idx holds valid entries in its first n_outliers slots.
    """
    _f16_dev(X, "X")
    s, h = X.shape
    dev = X.device
    lib = load_library()
    Xq = torch.empty((s, h), dtype=torch.int8, device=dev)
    ax = torch.empty((s,), dtype=torch.float32, device=dev)
    flags = torch.empty((h,), dtype=torch.uint8, device=dev)
    idx = torch.empty((h,), dtype=torch.int32, device=dev)
    n = torch.empty((1,), dtype=torch.int32, device=dev)
    nb = int(lib.llmint8_quantize_rows_scratch_size(h))
    scratch = torch.empty(max(nb, 256), dtype=torch.uint8, device=dev)
    _check("llmint8_quantize_rows_ex", lib.llmint8_quantize_rows_ex(
        _ptr(X), s, h, float(alpha), int(x_scale), _ptr(Xq), _ptr(ax),
        _ptr(flags), _ptr(idx), _ptr(n), _ptr(scratch), nb, _stream(stream)))
    return Xq, ax, flags, idx, n


def llmint8_matmul(X: torch.Tensor, w: PreparedWeight, alpha: float = 6.0,
                   out: Optional[torch.Tensor] = None,
                   workspace: Optional[Workspace] = None,
                   ci: Optional[torch.Tensor] = None, path: int = 0,
                   events=None, stream=None,
                   x_scale: int = SCALE_VECTORWISE,
                   status_host: Optional[HostStatusWord] = None,
                   wo_build: int = WO_SHARED) -> torch.Tensor:
    """C = LLM.int8()(X, W): X fp16 [s,h] on the GPU -> fp16 [s,o].

    ci (optional, int32 [s,o]) receives the exact int32 accumulators; path
    forces a kernel (PATH_*: prefill 1, decode 2, prefill with one CTA per
    tile 3, prefill with CTA pairs 4); events = (start, stop)
    torch.cuda.Event pair recorded around the GEMM kernel; x_scale =
    SCALE_TENSORWISE quantises X with one constant for the whole tensor;
    status_host (a HostStatusWord) reports device anomalies on the next call;
    wo_build picks where the fp16 outlier rows of W are built (WO_*).
    The workspace's max_outliers is passed along.
    """
    _f16_dev(X, "X")
    s, h = X.shape
    if h != w.h:
        raise ValueError(f"X has h={h}, weight has h={w.h}")
    if out is None:
        out = torch.empty((s, w.o), dtype=torch.float16, device=X.device)
    if workspace is None:
        workspace = Workspace(s, h, w.o, device=X.device)
    opts = llmint8_matmul_opts()
    opts.path = int(path)
    opts.x_scale = int(x_scale)
    opts.max_outliers = workspace.max_outliers
    opts.wo_build = int(wo_build)
    if status_host is not None:
        opts.status_host = status_host.t.data_ptr()
    if ci is not None:
        if ci.dtype != torch.int32 or ci.shape != (s, w.o):
            raise ValueError("ci must be int32 [s,o]")
        opts.ci_dev = ci.data_ptr()
    if events is not None:
        for e in events:  # torch creates its events lazily, on first record
            if not e.cuda_event:
                e.record(stream if stream is not None
                         else torch.cuda.current_stream())
        opts.gemm_event_start = events[0].cuda_event
        opts.gemm_event_stop = events[1].cuda_event
    _check("llmint8_matmul_ex", load_library().llmint8_matmul_ex(
        _ptr(X), s, ctypes.byref(w.c), float(alpha), _ptr(out),
        _ptr(workspace.buf), workspace.nbytes, ctypes.byref(opts),
        _stream(stream)))
    llmint8_matmul.last_launches = int(opts.launches)
    return out


def llmint8_matmul_noalloc(X: torch.Tensor, w: PreparedWeight,
                           alpha: float = 6.0,
                           out: Optional[torch.Tensor] = None,
                           stream=None) -> torch.Tensor:
    """llmint8_matmul without a caller workspace: the library's own static
    device scratch is used instead (see include/llmint8.h for who needs this
    and its limits). Only `out` may be allocated here, by torch, when it is
    not given."""
    _f16_dev(X, "X")
    s, h = X.shape
    if h != w.h:
        raise ValueError(f"X has h={h}, weight has h={w.h}")
    if out is None:
        out = torch.empty((s, w.o), dtype=torch.float16, device=X.device)
    _check("llmint8_matmul_noalloc", load_library().llmint8_matmul_noalloc(
        _ptr(X), s, ctypes.byref(w.c), float(alpha), _ptr(out), _stream(stream)))
    return out


def llmint8_matmul_host(X_host: torch.Tensor, w: PreparedWeight,
                        alpha: float, out_host: torch.Tensor,
                        workspace: Workspace, stream=None,
                        x_scale: int = SCALE_VECTORWISE) -> torch.Tensor:
    """End-to-end form: host fp16 X in, host fp16 C out (synchronises)."""
    if X_host.is_cuda or out_host.is_cuda:
        raise ValueError("X_host and out_host must be host tensors")
    s, h = X_host.shape
    opts = llmint8_matmul_opts()
    opts.x_scale = int(x_scale)
    opts.max_outliers = workspace.max_outliers
    _check("llmint8_matmul_host_ex", load_library().llmint8_matmul_host_ex(
        _ptr(X_host), s, ctypes.byref(w.c), float(alpha), _ptr(out_host),
        _ptr(workspace.buf), workspace.nbytes, ctypes.byref(opts), _stream(stream)))
    return out_host


def llmint8_read_outlier_tiles(workspace: Workspace, s: Optional[int] = None,
                               stream=None, tiles: bool = True):
    """(n, XO [s,n] fp16, WO [n,o] fp16) of the last matmul on `workspace`,
    which had `s` rows (default: the row count the workspace was sized for;
    the workspace layout depends on it). tiles=False reads |O| alone."""
    h, o = workspace.h, workspace.o
    s = workspace.s if s is None else int(s)
    cap = workspace.max_outliers or h
    n = ctypes.c_int32(0)
    if not tiles:
        _check("llmint8_read_outlier_tiles_ex", load_library().llmint8_read_outlier_tiles_ex(
            _ptr(workspace.buf), workspace.nbytes, s, h, o, workspace.max_outliers,
            ctypes.byref(n), None, None, _stream(stream)))
        return n.value, None, None
    XO = torch.empty((s * cap,), dtype=torch.float16)
    WO = torch.empty((cap * o,), dtype=torch.float16)
    _check("llmint8_read_outlier_tiles_ex", load_library().llmint8_read_outlier_tiles_ex(
        _ptr(workspace.buf), workspace.nbytes, s, h, o, workspace.max_outliers,
        ctypes.byref(n), _ptr(XO), _ptr(WO), _stream(stream)))
    k = n.value
    if k > cap:  # the call kept no outlier tiles
        return k, None, None
    return k, XO[: s * k].view(s, k), WO[: k * o].view(k, o)


def llmint8_wait_selftest(workspace: Workspace, limit_ns: int = 2_000_000,
                          stream=None) -> None:
    """Enqueue the bounded-wait self-test (its waits run out by design)."""
    _check("llmint8_wait_selftest", load_library().llmint8_wait_selftest(
        _ptr(workspace.buf), workspace.nbytes, int(limit_ns), _stream(stream)))


def llmint8_noalloc_read_device_status(stream=None) -> int:
    """Status bits of the allocation-free entry point on the current device
    (read and cleared; its state block is cleared too)."""
    bits = ctypes.c_int32(0)
    rc = load_library().llmint8_noalloc_read_device_status(ctypes.byref(bits),
                                                           _stream(stream))
    if rc not in (OK, -6):
        _check("llmint8_noalloc_read_device_status", rc)
    return bits.value


def llmint8_read_device_status(workspace: Workspace, stream=None) -> int:
    bits = ctypes.c_int32(0)
    rc = load_library().llmint8_read_device_status(
        _ptr(workspace.buf), workspace.nbytes, ctypes.byref(bits), _stream(stream))
    if rc not in (OK, -6):
        _check("llmint8_read_device_status", rc)
    return bits.value


_cudart = None


def event_elapsed_ms(start, stop) -> float:
    """Milliseconds between two torch.cuda.Event objects recorded by the
    library (torch's own elapsed_time only accepts events torch recorded)."""
    global _cudart
    if _cudart is None:
        cand = os.path.join(os.path.dirname(torch.__file__), "..", "nvidia",
                            "cuda_runtime", "lib", "libcudart.so.12")
        _cudart = ctypes.CDLL(cand if os.path.exists(cand) else "libcudart.so.12")
        _cudart.cudaEventElapsedTime.argtypes = [ctypes.POINTER(ctypes.c_float),
                                                 _vp, _vp]
        _cudart.cudaEventElapsedTime.restype = ctypes.c_int
    ms = ctypes.c_float(0.0)
    rc = _cudart.cudaEventElapsedTime(ctypes.byref(ms), _vp(start.cuda_event),
                                      _vp(stop.cuda_event))
    if rc != 0:
        raise RuntimeError(f"cudaEventElapsedTime failed ({rc})")
    return float(ms.value)


def effective_tops(s: int, h: int, o: int, seconds: float) -> float:
    return 2.0 * s * h * o / seconds / 1e12 if seconds > 0 else math.nan
