"""Mixed-precision MoE experts served from paged 3/4/8-bit weights on B200.

A thin ctypes binding over ``libmpe.so`` (C ABI declared in ``include/mpe.h``).
This module only marshals arguments: every step of the path -- allocation,
absmax, scaling, encoding, packing, routing, the expert FFN and the combine --
runs in the library's CUDA kernels. PyTorch supplies device memory and the
current stream. There is no CPU fallback: if the library is missing the
import of any entry point raises.

Method: PagedWeight ("PagedWeight: Efficient MoE LLM Serving with Dynamic
Quality-Aware Weight Quantization"), see include/mpe.h for each call's
contract and citation.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmpe.so")

MPE_OK = 0
ERRORS = {
    -1: "MPE_ERR_INVALID", -2: "MPE_ERR_INFEASIBLE", -3: "MPE_ERR_STATE_CAP",
    -4: "MPE_ERR_POOL", -5: "MPE_ERR_CUDA", -6: "MPE_ERR_ORDER", -7: "MPE_ERR_DEVICE",
}
STATUS_BAD_EXPERT_ID = 0x1
STATUS_NONFINITE = 0x2
STATUS_WAIT_TIMEOUT = 0x4
PATH_AUTO, PATH_DECODE, PATH_PREFILL = 0, 1, 2
ALLOCATOR_EXACT, ALLOCATOR_PROPORTIONAL, ALLOCATOR_MEASURED = 0, 1, 2
STORE_DEVICE, STORE_HOST = 0, 1
MAX_COMP_CHANNELS = 256
ALLOC_STATE_CAP = 65536
MAX_EXPERTS = 1024

# every symbol include/mpe.h declares
EXPORTS = [
    "mpe_create", "mpe_destroy", "mpe_set_stream", "mpe_set_path", "mpe_allocate_bits",
    "mpe_allocate_bits_proportional", "mpe_allocate_bits_table", "mpe_set_allocator",
    "mpe_measure_loss", "mpe_repage_async", "mpe_repage_commit", "mpe_set_compensation",
    "mpe_select_salient", "mpe_get_kept_channels", "mpe_prefix_create", "mpe_prefix_destroy",
    "mpe_prefix_last_error", "mpe_prefix_quantize", "mpe_prefix_repage", "mpe_prefix_moe_ffn",
    "mpe_prefix_read_layer", "mpe_prefix_get_absmax", "mpe_selftest_wait",
    "mpe_quantize_experts", "mpe_repage", "mpe_moe_ffn", "mpe_moe_ffn_host", "mpe_route",
    "mpe_get_page_table", "mpe_expert_stream_bytes", "mpe_read_expert_packed",
    "mpe_get_scales", "mpe_get_bits", "mpe_get_status", "mpe_last_error",
    "mpe_last_error_global", "mpe_kernel_launches", "mpe_version", "mpe_profile_enable",
    "mpe_profile_read", "mpe_route_noalloc", "mpe_moe_ffn_host_async", "mpe_host_wait",
]
PROFILE_SLOTS = ["route", "gate_up", "swiglu_reduce", "down", "combine", "tc_gate_up",
                 "tc_down", "tc_permute", "select", "compensate"]


class MpeError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{ERRORS.get(code, code)}: {msg}")
        self.code = code


class Config(ctypes.Structure):
    _fields_ = [("E", ctypes.c_int32), ("H", ctypes.c_int32), ("F", ctypes.c_int32),
                ("page_bytes", ctypes.c_uint32), ("pool_pages", ctypes.c_uint32),
                ("device", ctypes.c_int32), ("path", ctypes.c_int32),
                ("reserved", ctypes.c_int32), ("stream", ctypes.c_void_p)]


class Pte(ctypes.Structure):
    _fields_ = [("bits", ctypes.c_uint8), ("pad", ctypes.c_uint8 * 3),
                ("scale", ctypes.c_float), ("first", ctypes.c_uint32),
                ("n_pages", ctypes.c_uint32)]


PTE_DTYPE = np.dtype([("bits", np.uint8), ("pad", np.uint8, 3), ("scale", np.float32),
                      ("first", np.uint32), ("n_pages", np.uint32)])

_lib = None


def lib() -> ctypes.CDLL:
    """Load libmpe.so (raises if it was not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m mixed_precision_expert_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, u32, u64, sz = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_uint32,
                             ctypes.c_uint64, ctypes.c_size_t)
    sig = {
        "mpe_create": (i32, [ctypes.POINTER(vp), ctypes.POINTER(Config)]),
        "mpe_destroy": (None, [vp]),
        "mpe_set_stream": (i32, [vp, vp]),
        "mpe_set_path": (i32, [vp, i32]),
        "mpe_allocate_bits": (i32, [vp, vp, i32, u64, vp]),
        "mpe_allocate_bits_proportional": (i32, [vp, vp, i32, u64, vp]),
        "mpe_allocate_bits_table": (i32, [vp, vp, vp, i32, u64, vp]),
        "mpe_measure_loss": (i32, [vp, vp]),
        "mpe_set_compensation": (i32, [vp, i32, i32]),
        "mpe_select_salient": (i32, [vp, i32, i32, i32, vp, vp]),
        "mpe_get_kept_channels": (i32, [vp, i32, vp, sz]),
        "mpe_prefix_create": (i32, [ctypes.POINTER(vp), ctypes.POINTER(Config)]),
        "mpe_prefix_destroy": (None, [vp]),
        "mpe_prefix_last_error": (ctypes.c_char_p, [vp]),
        "mpe_prefix_quantize": (i32, [vp, vp, vp]),
        "mpe_prefix_repage": (i32, [vp, vp, ctypes.POINTER(u64)]),
        "mpe_prefix_moe_ffn": (i32, [vp, vp, i32, vp, vp, i32, vp]),
        "mpe_prefix_read_layer": (i32, [vp, i32, i32, vp, sz]),
        "mpe_prefix_get_absmax": (i32, [vp, vp]),
        "mpe_selftest_wait": (i32, [vp, u64]),
        "mpe_set_allocator": (i32, [vp, i32]),
        "mpe_repage_async": (i32, [vp, u64, vp, vp]),
        "mpe_repage_commit": (i32, [vp, i32, vp]),
        "mpe_quantize_experts": (i32, [vp, vp, vp]),
        "mpe_repage": (i32, [vp, u64, vp, vp]),
        "mpe_moe_ffn": (i32, [vp, vp, i32, vp, vp, i32, vp]),
        "mpe_moe_ffn_host": (i32, [vp, vp, i32, vp, vp, i32, vp]),
        "mpe_moe_ffn_host_async": (i32, [vp, vp, i32, vp, vp, i32, vp, vp]),
        "mpe_host_wait": (i32, [vp, u64]),
        "mpe_route": (i32, [vp, vp, i32, i32, vp, vp, vp]),
        "mpe_get_page_table": (i32, [vp, vp, vp, sz]),
        "mpe_expert_stream_bytes": (sz, [vp, i32]),
        "mpe_read_expert_packed": (i32, [vp, i32, vp, sz]),
        "mpe_get_scales": (i32, [vp, vp, vp]),
        "mpe_get_bits": (i32, [vp, vp]),
        "mpe_get_status": (i32, [vp, vp, i32]),
        "mpe_last_error": (ctypes.c_char_p, [vp]),
        "mpe_last_error_global": (ctypes.c_char_p, []),
        "mpe_kernel_launches": (u64, [vp]),
        "mpe_version": (i32, []),
        "mpe_profile_enable": (i32, [vp, i32]),
        "mpe_profile_read": (i32, [vp, vp, vp, i32, i32]),
        "mpe_route_noalloc": (i32, [vp, i32, i32, i32, vp, vp, vp, vp]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    _lib = L
    return L


def _ptr(a) -> int:
    if a is None:
        return 0
    if hasattr(a, "data_ptr"):
        return a.data_ptr()
    if isinstance(a, np.ndarray):
        return a.ctypes.data
    raise TypeError(type(a))


def _check(rc: int, ctx=None):
    if rc != MPE_OK:
        L = lib()
        msg = (L.mpe_last_error(ctx) if ctx else L.mpe_last_error_global()) or b""
        raise MpeError(rc, msg.decode())


def _stream() -> int:
    import torch
    return torch.cuda.current_stream().cuda_stream


def allocate_bits(p, W, B: int) -> np.ndarray:
    """b_e in {3,4,8} minimising sum p_e L(b_e) s.t. sum b_e W_e <= B (device DP)."""
    p = np.ascontiguousarray(p, dtype=np.float64)
    W = np.ascontiguousarray(W, dtype=np.uint64)
    out = np.zeros(len(p), dtype=np.uint8)
    _check(lib().mpe_allocate_bits(_ptr(p), _ptr(W), len(p), int(B), _ptr(out)))
    return out


def allocate_bits_proportional(p, W, B: int) -> np.ndarray:
    """The page's proportional rule (budget share by importance, rounded up to
    3/4/8 bits) with the library's budget repair (device kernel)."""
    p = np.ascontiguousarray(p, dtype=np.float64)
    W = np.ascontiguousarray(W, dtype=np.uint64)
    out = np.zeros(len(p), dtype=np.uint8)
    _check(lib().mpe_allocate_bits_proportional(_ptr(p), _ptr(W), len(p), int(B), _ptr(out)))
    return out


def allocate_bits_table(p, loss, W, B: int) -> np.ndarray:
    """The exact program with a loss per expert and width (float64[E, 3],
    columns 3, 4, 8 bits), e.g. Context.measure_loss() (device DP)."""
    p = np.ascontiguousarray(p, dtype=np.float64)
    loss = np.ascontiguousarray(loss, dtype=np.float64)
    W = np.ascontiguousarray(W, dtype=np.uint64)
    if loss.shape != (len(p), 3):
        raise ValueError("loss must be float64[E, 3]")
    out = np.zeros(len(p), dtype=np.uint8)
    _check(lib().mpe_allocate_bits_table(_ptr(p), _ptr(loss), _ptr(W), len(p), int(B),
                                         _ptr(out)))
    return out


def select_salient(rows, n: int, out=None):
    """Per row of a bf16 CUDA matrix [rows, cols]: the n channels of largest
    magnitude (ties to the lower index), ascending; int32 [rows, n] (a row's
    first min(n, cols) entries). Current stream."""
    import torch
    R, C = rows.shape
    if out is None:
        out = torch.full((R, n), -1, dtype=torch.int32, device=rows.device)
    _check(lib().mpe_select_salient(_ptr(rows), R, C, n, _ptr(out), _stream()))
    return out


def route_noalloc(ids, E: int, perm, offsets, inv):
    """Bucketing into caller-provided device buffers without any device
    allocation (mpe_route_noalloc); runs on the current stream."""
    T, k = ids.shape
    _check(lib().mpe_route_noalloc(_ptr(ids), T, k, E, _ptr(perm), _ptr(offsets), _ptr(inv),
                                   _stream()))


class Context:
    """One MoE layer's paged experts on one GPU (wraps an ``mpe_ctx``)."""

    def __init__(self, E: int, H: int, F: int, page_bytes: int = 0, pool_pages: int = 0,
                 device: int | None = None, path: int = PATH_AUTO):
        import torch
        L = lib()
        dev = torch.cuda.current_device() if device is None else device
        cfg = Config(E, H, F, page_bytes, pool_pages, dev, path, 0, None)
        h = ctypes.c_void_p()
        _check(L.mpe_create(ctypes.byref(h), ctypes.byref(cfg)))
        self._h = h
        self.E, self.H, self.F = E, H, F
        self._masters = None

    def close(self):
        if getattr(self, "_h", None):
            lib().mpe_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def _sync_stream(self):
        _check(lib().mpe_set_stream(self._h, _stream()), self._h)

    def set_path(self, path: int):
        _check(lib().mpe_set_path(self._h, path), self._h)

    def set_allocator(self, allocator: int):
        """ALLOCATOR_EXACT (default), ALLOCATOR_PROPORTIONAL or ALLOCATOR_MEASURED
        for later repages."""
        _check(lib().mpe_set_allocator(self._h, allocator), self._h)

    def set_compensation(self, n_channels: int, store: int = STORE_DEVICE):
        """Compensate the n_channels salient input channels of every projection
        on the streaming path (0: off); the residual store in device memory
        (STORE_DEVICE) or mapped host memory (STORE_HOST)."""
        self._sync_stream()
        _check(lib().mpe_set_compensation(self._h, int(n_channels), int(store)), self._h)

    def kept_channels(self, which: int, rows: int, n: int) -> np.ndarray:
        """int32 [rows, n]: the last compensated forward's kept channels of x
        (which 0, rows = T) or of h (which 1, rows = T k, by route position)."""
        out = np.zeros((rows, n), dtype=np.int32)
        _check(lib().mpe_get_kept_channels(self._h, which, _ptr(out), out.size), self._h)
        return out

    def selftest_wait(self, limit_ns: int):
        """A device wait that nothing completes gives up after limit_ns and sets
        STATUS_WAIT_TIMEOUT (the failure path of every bounded wait)."""
        self._sync_stream()
        _check(lib().mpe_selftest_wait(self._h, int(limit_ns)), self._h)

    def measure_loss(self) -> np.ndarray:
        """float64[E, 3]: each expert's measured quantization MSE at 3, 4, 8 bits."""
        self._sync_stream()
        out = np.zeros((self.E, 3), dtype=np.float64)
        _check(lib().mpe_measure_loss(self._h, _ptr(out)), self._h)
        return out

    def quantize_experts(self, masters, bits):
        """masters: E flat fp16 CUDA tensors (W1 | W3 | W2); bits: uint8[E]."""
        self._sync_stream()
        assert len(masters) == self.E
        arr = (ctypes.c_void_p * self.E)(*[m.data_ptr() for m in masters])
        b = np.ascontiguousarray(bits, dtype=np.uint8)
        self._masters = list(masters)  # the library borrows them
        _check(lib().mpe_quantize_experts(self._h, arr, _ptr(b)), self._h)

    def repage(self, B: int, p) -> int:
        self._sync_stream()
        p = np.ascontiguousarray(p, dtype=np.float64)
        n = ctypes.c_int32(0)
        _check(lib().mpe_repage(self._h, int(B), _ptr(p), ctypes.byref(n)), self._h)
        return n.value

    def repage_async(self, B: int, p) -> int:
        """Start an overlapped repage (forward passes keep the current pages
        until repage_commit); returns the number of experts changed."""
        self._sync_stream()
        p = np.ascontiguousarray(p, dtype=np.float64)
        n = ctypes.c_int32(0)
        _check(lib().mpe_repage_async(self._h, int(B), _ptr(p), ctypes.byref(n)), self._h)
        return n.value

    def repage_commit(self, wait: bool = True) -> bool:
        """Switch to the pending repage's pages (wait=False: only if ready)."""
        self._sync_stream()
        done = ctypes.c_int32(0)
        _check(lib().mpe_repage_commit(self._h, 1 if wait else 0, ctypes.byref(done)), self._h)
        return bool(done.value)

    def moe_ffn(self, x, ids, w, out=None):
        import torch
        self._sync_stream()
        T, k = ids.shape
        if out is None:
            out = torch.empty((T, self.H), dtype=torch.bfloat16, device=x.device)
        _check(lib().mpe_moe_ffn(self._h, _ptr(x), T, _ptr(ids), _ptr(w), k, _ptr(out)),
               self._h)
        return out

    def moe_ffn_host(self, x, ids, w, out):
        """Host (pinned) buffers in, host buffer out; synchronous."""
        self._sync_stream()
        T, k = ids.shape
        _check(lib().mpe_moe_ffn_host(self._h, _ptr(x), T, _ptr(ids), _ptr(w), k, _ptr(out)),
               self._h)
        return out

    def moe_ffn_host_async(self, x, ids, w, out) -> int:
        """Host (pinned) buffers in, host buffer out; queued, returns a ticket.
        The buffers belong to the library until wait_host(ticket) returns."""
        self._sync_stream()
        T, k = ids.shape
        t = ctypes.c_uint64(0)
        _check(lib().mpe_moe_ffn_host_async(self._h, _ptr(x), T, _ptr(ids), _ptr(w), k,
                                             _ptr(out), ctypes.byref(t)), self._h)
        return t.value

    def wait_host(self, ticket: int):
        _check(lib().mpe_host_wait(self._h, ctypes.c_uint64(ticket)), self._h)

    def route(self, ids):
        import torch
        self._sync_stream()
        T, k = ids.shape
        n = T * k
        perm = torch.empty(max(n, 1), dtype=torch.int32, device=ids.device)
        inv = torch.empty(max(n, 1), dtype=torch.int32, device=ids.device)
        offs = torch.empty(self.E + 1, dtype=torch.int32, device=ids.device)
        _check(lib().mpe_route(self._h, _ptr(ids), T, k, _ptr(perm), _ptr(offs), _ptr(inv)),
               self._h)
        return perm[:n], offs, inv[:n]

    def page_table(self):
        pte = np.zeros(self.E, dtype=PTE_DTYPE)
        _check(lib().mpe_get_page_table(self._h, _ptr(pte), None, 0), self._h)
        total = int(pte["n_pages"].sum())
        pidx = np.zeros(max(total, 1), dtype=np.uint32)
        _check(lib().mpe_get_page_table(self._h, None, _ptr(pidx), len(pidx)), self._h)
        return pte, pidx[:total]

    def expert_stream(self, e: int) -> np.ndarray:
        n = lib().mpe_expert_stream_bytes(self._h, e)
        out = np.zeros(n, dtype=np.uint8)
        _check(lib().mpe_read_expert_packed(self._h, e, _ptr(out), n), self._h)
        return out

    def scales(self):
        s = np.zeros(self.E, dtype=np.float32)
        m = np.zeros(self.E, dtype=np.float32)
        _check(lib().mpe_get_scales(self._h, _ptr(s), _ptr(m)), self._h)
        return s, m

    def bits(self) -> np.ndarray:
        b = np.zeros(self.E, dtype=np.uint8)
        _check(lib().mpe_get_bits(self._h, _ptr(b)), self._h)
        return b

    def status(self, clear: bool = False) -> int:
        st = np.zeros(1, dtype=np.uint32)
        _check(lib().mpe_get_status(self._h, _ptr(st), 1 if clear else 0), self._h)
        return int(st[0])

    def kernel_launches(self) -> int:
        return int(lib().mpe_kernel_launches(self._h))

    def profile(self, enable: bool):
        """Record CUDA events around each forward-pass kernel (device times)."""
        _check(lib().mpe_profile_enable(self._h, 1 if enable else 0), self._h)

    def profile_read(self, reset: bool = True) -> dict:
        """{slot: (total ms, launches)} for the recorded kernels."""
        n = len(PROFILE_SLOTS)
        ms = np.zeros(n, dtype=np.float64)
        cnt = np.zeros(n, dtype=np.int64)
        _check(lib().mpe_profile_read(self._h, _ptr(ms), _ptr(cnt), n, 1 if reset else 0),
               self._h)
        return {name: (float(ms[i]), int(cnt[i])) for i, name in enumerate(PROFILE_SLOTS)}


class PrefixStore:
    """The prefix-compatible variant (mpe_prefix_*): nested-grid codes stored in
    layers A (3 bits), B (1 bit), C (4 bits); a width change drops or adds
    layers."""

    LAYER_BITS = (3, 1, 4)

    def __init__(self, E: int, H: int, F: int, page_bytes: int = 0, pool_pages: int = 0,
                 device: int | None = None):
        import torch
        L = lib()
        dev = torch.cuda.current_device() if device is None else device
        cfg = Config(E, H, F, page_bytes, pool_pages, dev, 0, 0,
                     torch.cuda.current_stream().cuda_stream)
        h = ctypes.c_void_p()
        _check(L.mpe_prefix_create(ctypes.byref(h), ctypes.byref(cfg)))
        self._h = h
        self.E, self.H, self.F = E, H, F
        self._masters = None

    def _check(self, rc):
        if rc != 0:
            msg = lib().mpe_prefix_last_error(self._h)
            raise MpeError(rc, msg.decode() if msg else "")

    def close(self):
        if getattr(self, "_h", None):
            lib().mpe_prefix_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def quantize(self, masters, bits):
        arr = (ctypes.c_void_p * self.E)(*[m.data_ptr() for m in masters])
        b = np.ascontiguousarray(bits, dtype=np.uint8)
        self._masters = list(masters)
        self._check(lib().mpe_prefix_quantize(self._h, arr, _ptr(b)))

    def repage(self, bits) -> int:
        """New widths; returns the bytes the change moved."""
        b = np.ascontiguousarray(bits, dtype=np.uint8)
        moved = ctypes.c_uint64(0)
        self._check(lib().mpe_prefix_repage(self._h, _ptr(b), ctypes.byref(moved)))
        return int(moved.value)

    def moe_ffn(self, x, ids, w, out=None):
        import torch
        T, k = ids.shape
        if out is None:
            out = torch.empty((T, self.H), dtype=torch.bfloat16, device=x.device)
        self._check(lib().mpe_prefix_moe_ffn(self._h, _ptr(x), T, _ptr(ids), _ptr(w), k,
                                             _ptr(out)))
        return out

    def read_layer(self, e: int, layer: int) -> np.ndarray:
        """Layer `layer` (0 A, 1 B, 2 C) of expert e: its chunk stream, uint8."""
        n = 3 * self.H * self.F * self.LAYER_BITS[layer] // 8
        out = np.zeros(n, dtype=np.uint8)
        self._check(lib().mpe_prefix_read_layer(self._h, e, layer, _ptr(out), out.nbytes))
        return out

    def absmax(self) -> np.ndarray:
        out = np.zeros(self.E, dtype=np.float32)
        self._check(lib().mpe_prefix_get_absmax(self._h, _ptr(out)))
        return out
