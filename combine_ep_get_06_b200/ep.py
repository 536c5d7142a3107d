"""Python binding of libep_b200.so (include/ep.h): argument marshalling only.

Every step of dispatch / combine runs in the library's CUDA kernels; torch
only supplies device memory and the current stream.  There is no CPU path:
if the library is missing or cannot be loaded, every call raises.

The call shapes follow the DeepEP V2 README, section "Interfaces and
examples": dispatch takes x (bf16, or an FP8 (data, scale_factors) tuple),
topk_idx (-1 = dropped slot), topk_weights, num_experts and
expert_alignment, and returns recv_x, recv_topk_idx, recv_topk_weights and
a handle; combine takes expert outputs and the handle; the backward of
dispatch is a combine and the backward of combine is a dispatch.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple, Union

import torch

from . import build as _build

EP_OK, EP_ERR_INVALID_ARG, EP_ERR_DEVICE, EP_ERR_CUDA = 0, 1, 2, 3
EP_X_BF16, EP_X_FP8, EP_X_BF16_TO_FP8, EP_X_BF16_TO_NVFP4 = 0, 1, 2, 3
EP_DEVERR_BAD_TOPK_IDX, EP_DEVERR_CAPACITY, EP_DEVERR_TIMEOUT, EP_DEVERR_CHECK = 1, 2, 4, 8


class EPError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(message)
        self.status = status


class _HandleC(ctypes.Structure):
    _fields_ = [(name, ctypes.c_int32) for name in
                ("num_tokens", "num_topk", "num_experts", "num_segments", "expert_alignment",
                 "max_recv_rows")] + \
               [(name, ctypes.c_void_p) for name in
                ("counts", "recv_counts", "offsets", "seg_tokens", "slot_map", "recv_src",
                 "pad_rows", "num_pad_rows", "error_word")]


class _GeomC(ctypes.Structure):
    """ep_mgpu_geometry (include/ep_multi.h)."""
    _fields_ = [(name, ctypes.c_int32) for name in
                ("rank", "world", "max_tokens", "num_topk", "num_experts", "expert_alignment", "hidden",
                 "x_mode", "experts_per_rank", "max_recv_rows", "row_bytes", "scale_bytes")] + \
               [(name, ctypes.c_int64) for name in
                ("off_recv_x", "off_recv_scales", "off_recv_src", "off_recv_topk_idx",
                 "off_recv_topk_weights", "off_y", "off_all_counts", "off_dest", "off_raw_counts",
                 "off_recv_counts", "off_recv_offsets", "off_num_pad_rows", "off_error_word",
                 "block_bytes")]


_LIB = None

# name -> (restype, argtypes); mirrors include/ep.h
_P, _I32, _SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
_HP = ctypes.POINTER(_HandleC)
_GP = ctypes.POINTER(_GeomC)
SIGNATURES = {
    "ep_abi_version": (_I32, []),
    "ep_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "ep_last_error": (ctypes.c_char_p, []),
    "ep_set_num_sms": (ctypes.c_int, [_I32]),
    "ep_get_num_sms": (_I32, []),
    "ep_max_recv_rows": (_I32, [_I32, _I32, _I32, _I32]),
    "ep_handle_bytes": (_SZ, [_I32, _I32, _I32, _I32, _I32, _I32]),
    "ep_handle_init": (ctypes.c_int, [_HP, _I32, _I32, _I32, _I32, _I32, _I32, _P, _SZ]),
    "ep_layout_workspace_bytes": (_SZ, [_HP]),
    "ep_get_layout": (ctypes.c_int, [_HP, _P, _I32, _P, _P, _P, _P, _SZ, _P]),
    "ep_get_layout_static": (ctypes.c_int, [_HP, _P, _I32, _P, _P, _P, _P]),
    "ep_dispatch": (ctypes.c_int, [_HP, ctypes.c_int, _P, _P, _I32, _P, _P, _P]),
    "ep_layout_dispatch": (ctypes.c_int, [_HP, _P, _I32, _P, _P, _P, _P, _SZ, ctypes.c_int, _P, _P, _I32,
                                          _P, _P, _P]),
    "ep_combine": (ctypes.c_int, [_HP, _P, _I32, _P, _P, _P, _P, _P]),
    "ep_combine_backward": (ctypes.c_int, [_HP, _P, _P, _I32, _P, _P, _P, _P]),
    "ep_combine_fp8": (ctypes.c_int, [_HP, _P, _P, _I32, _P, _P, _P]),
    "ep_dispatch_mn_scales": (ctypes.c_int, [_HP, ctypes.c_int, _P, _P, _I32, _P, _P, _I32, _P]),
    "ep_read_recv_counts": (ctypes.c_int, [_HP, _P, _P]),
    "ep_read_total_rows": (ctypes.c_int, [_HP, ctypes.POINTER(_I32), _P]),
    "ep_check_error": (ctypes.c_int, [_HP, ctypes.POINTER(ctypes.c_uint32), _P]),
    # include/ep_multi.h
    "ep_mgpu_geometry_init": (ctypes.c_int, [_GP, _I32, _I32, _I32, _I32, _I32, _I32, _I32, ctypes.c_int]),
    "ep_mgpu_block_alloc": (ctypes.c_int, [_SZ, ctypes.POINTER(_P)]),
    "ep_mgpu_block_free": (ctypes.c_int, [_P]),
    "ep_ipc_export": (ctypes.c_int, [_P, _P]),
    "ep_ipc_import": (ctypes.c_int, [_P, ctypes.POINTER(_P)]),
    "ep_ipc_close": (ctypes.c_int, [_P]),
    "ep_mgpu_dispatch": (ctypes.c_int, [_GP, _HP, _P, _I32, _P, ctypes.c_int, _P, _P, _P, _P, _P]),
    "ep_mgpu_combine": (ctypes.c_int, [_GP, _HP, _P, _P, _P, _P, _P]),
    "ep_mgpu_read_total_rows": (ctypes.c_int, [_GP, _P, ctypes.POINTER(_I32), _P]),
    "ep_mgpu_check_error": (ctypes.c_int, [_GP, _P, ctypes.POINTER(ctypes.c_uint32), _P]),
}


def _checked() -> bool:
    """EP_CHECKED=1 in the environment selects the checked build."""
    return os.environ.get("EP_CHECKED", "0") not in ("", "0")


def library_path() -> str:
    return _build.CHECKED_LIB if _checked() else _build.LIB


def lib() -> ctypes.CDLL:
    """The loaded CUDA library; builds it first if the sources are newer."""
    global _LIB
    if _LIB is None:
        checked = _checked()
        path = library_path()
        if not _build.up_to_date(checked):
            try:
                _build.build(checked=checked)
            except Exception as exc:  # no toolkit: fail loudly, there is no fallback
                if not os.path.exists(path):
                    raise RuntimeError(f"{os.path.basename(path)} is not built and cannot be built: {exc}")
        L = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = L
    return _LIB


def set_num_sms(num_sms: int) -> None:
    """SM budget of this host thread (DeepEP V2 README, "Interfaces and
    examples": num_sms): the dispatch and combine kernels launched from now
    on occupy at most num_sms SMs, leaving the rest to a kernel running
    beside them on another stream.  0 (the default) lets them take every
    SM."""
    _check(lib().ep_set_num_sms(int(num_sms)), "set_num_sms")


def get_num_sms() -> int:
    """This host thread's SM budget (0 = none)."""
    return int(lib().ep_get_num_sms())


class sm_budget:
    """Context manager: ``with ep.sm_budget(24): ...`` runs the body's
    dispatch / combine calls on at most 24 SMs, then restores the previous
    budget."""

    def __init__(self, num_sms: int):
        self.num_sms = int(num_sms)
        self.prev = 0

    def __enter__(self):
        self.prev = get_num_sms()
        set_num_sms(self.num_sms)
        return self

    def __exit__(self, *exc):
        set_num_sms(self.prev)
        return False


def _check(status: int, what: str):
    if status != EP_OK:
        L = lib()
        msg = L.ep_last_error().decode() or L.ep_status_string(status).decode()
        raise EPError(status, f"{what}: {msg}")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _stream(device: torch.device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _aligned_bytes(nbytes: int, device, zero: bool = False) -> Tuple[torch.Tensor, int]:
    buf = (torch.zeros if zero else torch.empty)(nbytes + 256, dtype=torch.uint8, device=device)
    return buf, (-buf.data_ptr()) % 256


def _need(t: torch.Tensor, name: str, dtypes, device=None, ndim=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a tensor")
    if t.dtype not in dtypes:
        raise TypeError(f"{name} has dtype {t.dtype}, expected one of {dtypes}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims")


def max_recv_rows(num_tokens: int, num_topk: int, num_experts: int, expert_alignment: int = 1) -> int:
    n = lib().ep_max_recv_rows(num_tokens, num_topk, num_experts, expert_alignment)
    if n < 0:
        raise ValueError("bad shape for max_recv_rows")
    return n


class EPHandle:
    """Routing metadata of one layout: device tensors carved from one block.

    counts [E] (c_e), num_recv_tokens_per_expert [E] (A(c_e), the per-expert
    row counts a grouped GEMM consumes), offsets [E+1], seg_tokens [S],
    slot_map [T*k], recv_src [max_recv_rows], pad_rows, num_pad_rows [1].
    Reusable for dispatch / combine with the same routing."""

    def __init__(self, num_tokens: int, num_topk: int, num_experts: int, num_segments: int = 1,
                 expert_alignment: int = 1, max_recv_rows: Optional[int] = None, device=None):
        L = lib()
        device = torch.device("cuda") if device is None else torch.device(device)
        if device.type == "cuda" and device.index is None:
            device = torch.device("cuda", torch.cuda.current_device())
        if max_recv_rows is None:
            max_recv_rows = L.ep_max_recv_rows(num_tokens, num_topk, num_experts, expert_alignment)
        nbytes = L.ep_handle_bytes(num_tokens, num_topk, num_experts, num_segments,
                                   expert_alignment, max_recv_rows)
        self.c = _HandleC()
        self.device = device
        if nbytes == 0:
            # let ep_handle_init produce the message
            _check(L.ep_handle_init(ctypes.byref(self.c), num_tokens, num_topk, num_experts,
                                    num_segments, expert_alignment, max_recv_rows, None, 0),
                   "EPHandle")
        self._block, off = _aligned_bytes(nbytes, device, zero=True)   # error word starts clear
        base = self._block.data_ptr() + off
        _check(L.ep_handle_init(ctypes.byref(self.c), num_tokens, num_topk, num_experts,
                                num_segments, expert_alignment, max_recv_rows, base, nbytes),
               "EPHandle")
        blk = self._block

        def view(ptr: int, n: int, dtype=torch.int32):
            o = ptr - blk.data_ptr()
            return blk[o: o + 4 * n].view(dtype)

        E, S = num_experts, num_segments
        self.counts = view(self.c.counts, E)
        self.num_recv_tokens_per_expert = view(self.c.recv_counts, E)
        self.offsets = view(self.c.offsets, E + 1)
        self.seg_tokens = view(self.c.seg_tokens, S)
        self.slot_map = view(self.c.slot_map, num_tokens * num_topk)
        self.recv_src = view(self.c.recv_src, max_recv_rows)
        self.pad_rows = view(self.c.pad_rows, max(1, E * (expert_alignment - 1)))
        self.num_pad_rows = view(self.c.num_pad_rows, 1)
        self.error_word = view(self.c.error_word, 1)
        ws = L.ep_layout_workspace_bytes(ctypes.byref(self.c))
        self._ws, self._ws_off = _aligned_bytes(ws, device)
        self.workspace_bytes = ws

    num_tokens = property(lambda s: s.c.num_tokens)
    num_topk = property(lambda s: s.c.num_topk)
    num_experts = property(lambda s: s.c.num_experts)
    num_segments = property(lambda s: s.c.num_segments)
    expert_alignment = property(lambda s: s.c.expert_alignment)
    max_recv_rows = property(lambda s: s.c.max_recv_rows)

    @property
    def workspace_ptr(self) -> int:
        return self._ws.data_ptr() + self._ws_off

    @property
    def ref(self):
        return ctypes.byref(self.c)

    def total_rows(self) -> int:
        """R = offsets[E] (synchronises the current stream)."""
        r = ctypes.c_int32(0)
        _check(lib().ep_read_total_rows(self.ref, ctypes.byref(r), _stream(self.device)), "total_rows")
        return r.value

    def recv_counts_host(self) -> list:
        """Rows of each expert, A(c_e), on the host (synchronises): the
        pages' num_recv_tokens_per_expert_list."""
        out = (ctypes.c_int32 * self.num_experts)()
        _check(lib().ep_read_recv_counts(self.ref, out, _stream(self.device)), "recv_counts_host")
        return list(out)

    def check_error(self) -> int:
        """Reads and clears the device error word; raises EPError if it was set."""
        bits = ctypes.c_uint32(0)
        _check(lib().ep_check_error(self.ref, ctypes.byref(bits), _stream(self.device)), "check_error")
        return bits.value


def get_layout(topk_idx: torch.Tensor, num_experts: int, *, num_segments: int = 1,
               expert_alignment: int = 1, topk_weights: Optional[torch.Tensor] = None,
               handle: Optional[EPHandle] = None, max_recv_rows: Optional[int] = None,
               recv_topk_idx: Optional[torch.Tensor] = None,
               recv_topk_weights: Optional[torch.Tensor] = None):
    """-> (handle, recv_topk_idx [max_recv_rows] int32, recv_topk_weights [max_recv_rows] f32)."""
    _need(topk_idx, "topk_idx", (torch.int64, torch.int32), ndim=2)
    T, k = topk_idx.shape
    dev = topk_idx.device
    if handle is None:
        handle = EPHandle(T, k, num_experts, num_segments, expert_alignment, max_recv_rows, device=dev)
    elif (handle.num_tokens, handle.num_topk, handle.num_experts) != (T, k, num_experts):
        raise ValueError("handle shape does not match topk_idx / num_experts")
    if topk_weights is not None:
        _need(topk_weights, "topk_weights", (torch.float32,), dev, 2)
        if tuple(topk_weights.shape) != (T, k):
            raise ValueError("topk_weights must have the shape of topk_idx")
    R = handle.max_recv_rows
    recv_idx = torch.empty(R, dtype=torch.int32, device=dev) if recv_topk_idx is None else recv_topk_idx
    recv_w = torch.empty(R, dtype=torch.float32, device=dev) if recv_topk_weights is None \
        else recv_topk_weights
    _need(recv_idx, "recv_topk_idx", (torch.int32,), dev, 1)
    _need(recv_w, "recv_topk_weights", (torch.float32,), dev, 1)
    if recv_idx.shape[0] != R or recv_w.shape[0] != R:
        raise ValueError("recv_topk_idx / recv_topk_weights must have max_recv_rows entries")
    _check(lib().ep_get_layout(handle.ref, topk_idx.data_ptr(), int(topk_idx.dtype == torch.int64),
                               _ptr(topk_weights), recv_idx.data_ptr(), recv_w.data_ptr(),
                               handle.workspace_ptr, handle.workspace_bytes, _stream(dev)),
           "get_layout")
    return handle, recv_idx, recv_w


XType = Union[torch.Tensor, Tuple[torch.Tensor, torch.Tensor]]


def _bf16_mode(use_fp8: bool, use_nvfp4: bool) -> int:
    if use_fp8 and use_nvfp4:
        raise ValueError("use_fp8 and use_nvfp4 are exclusive")
    return EP_X_BF16_TO_NVFP4 if use_nvfp4 else EP_X_BF16_TO_FP8 if use_fp8 else EP_X_BF16


def _dispatch_args(x: XType, handle: EPHandle, bf16_mode: int, recv_x, recv_scales, row_scales=True):
    """Checks x and the receive buffers (allocating those not given);
    returns (mode, x, x_scales, H, recv_x, recv_scales).  bf16_mode is the
    mode a bf16 x takes.  With row_scales False the row-major recv_scales
    is neither checked nor allocated."""
    dev = handle.device
    rows = handle.max_recv_rows
    x_scales = None
    if isinstance(x, (tuple, list)):
        x, x_scales = x
        _need(x, "x[0]", (torch.float8_e4m3fn, torch.uint8), dev, 2)
        _need(x_scales, "x[1]", (torch.float32,), dev, 2)
        mode = EP_X_FP8
    else:
        _need(x, "x", (torch.bfloat16,), dev, 2)
        mode = bf16_mode
    T, H = x.shape
    if T != handle.num_tokens:
        raise ValueError(f"x has {T} rows, handle has {handle.num_tokens} tokens")
    if mode == EP_X_FP8 and tuple(x_scales.shape) != (T, H // 128):
        raise ValueError("x scales must be [T, hidden/128]")
    if mode == EP_X_BF16:
        if recv_x is None:
            recv_x = torch.empty(rows, H, dtype=torch.bfloat16, device=dev)
        _need(recv_x, "recv_x", (torch.bfloat16,), dev, 2)
    elif mode == EP_X_BF16_TO_NVFP4:
        if H % 32 != 0:
            raise ValueError("NVFP4 dispatch needs hidden % 32 == 0")
        if recv_x is None:
            recv_x = torch.empty(rows, H // 2, dtype=torch.uint8, device=dev)
        _need(recv_x, "recv_x", (torch.uint8,), dev, 2)
        if tuple(recv_x.shape) != (rows, H // 2):
            raise ValueError("recv_x must be [max_recv_rows, hidden/2] in the NVFP4 mode")
        if recv_scales is None:
            recv_scales = torch.empty(rows, H // 16, dtype=torch.uint8, device=dev)
        _need(recv_scales, "recv_scales", (torch.uint8, torch.float8_e4m3fn), dev, 2)
        if tuple(recv_scales.shape) != (rows, H // 16):
            raise ValueError("recv_scales must be [max_recv_rows, hidden/16] in the NVFP4 mode")
        return mode, x, x_scales, H, recv_x, recv_scales
    else:
        if recv_x is None:
            recv_x = torch.empty(rows, H, dtype=torch.float8_e4m3fn, device=dev)
        _need(recv_x, "recv_x", (torch.float8_e4m3fn, torch.uint8), dev, 2)
        if row_scales:
            if recv_scales is None:
                recv_scales = torch.empty(rows, H // 128, dtype=torch.float32, device=dev)
            _need(recv_scales, "recv_scales", (torch.float32,), dev, 2)
            if tuple(recv_scales.shape) != (rows, H // 128):
                raise ValueError("recv_scales must be [max_recv_rows, hidden/128]")
    if tuple(recv_x.shape) != (rows, H):
        raise ValueError("recv_x must be [max_recv_rows, hidden]")
    return mode, x, x_scales, H, recv_x, recv_scales


def dispatch_with_handle(x: XType, handle: EPHandle, *, use_fp8: bool = False, use_nvfp4: bool = False,
                         recv_x: Optional[torch.Tensor] = None,
                         recv_scales: Optional[torch.Tensor] = None):
    """Dispatch with an existing handle (decode with a cached handle; the
    backward of combine).  x bf16 [T,H] -> recv_x bf16 [max_recv_rows,H];
    x bf16 with use_fp8 -> (recv_x e4m3 [rows,H], recv_scales f32 [rows,H/128]);
    x bf16 with use_nvfp4 -> (recv_x uint8 [rows,H/2] packed E2M1 pairs, the
    even element in the low nibble, recv_scales uint8 e4m3 [rows,H/16]);
    x = (x_fp8 [T,H], scales [T,H/128]) -> the same tuple, copied."""
    mode, x, x_scales, H, recv_x, recv_scales = _dispatch_args(x, handle, _bf16_mode(use_fp8, use_nvfp4),
                                                               recv_x, recv_scales)
    _check(lib().ep_dispatch(handle.ref, mode, x.data_ptr(), _ptr(x_scales), H, recv_x.data_ptr(),
                             _ptr(recv_scales), _stream(handle.device)), "dispatch")
    return recv_x if mode == EP_X_BF16 else (recv_x, recv_scales)


def dispatch(x: XType, topk_idx: Optional[torch.Tensor] = None,
             topk_weights: Optional[torch.Tensor] = None, num_experts: Optional[int] = None, *,
             expert_alignment: int = 1, num_segments: int = 1, handle: Optional[EPHandle] = None,
             use_fp8: bool = False, use_nvfp4: bool = False, max_recv_rows: Optional[int] = None,
             recv_x: Optional[torch.Tensor] = None, recv_scales: Optional[torch.Tensor] = None,
             recv_topk_idx: Optional[torch.Tensor] = None,
             recv_topk_weights: Optional[torch.Tensor] = None):
    """MoE dispatch.  With topk_idx: layout and dispatch in one call (the
    dispatch reads x while the layout runs); returns (recv_x, recv_topk_idx,
    recv_topk_weights, handle).  With only a handle (cached): returns
    (recv_x, None, None, handle)."""
    if topk_idx is None:
        if handle is None:
            raise ValueError("dispatch needs topk_idx or a handle")
        return dispatch_with_handle(x, handle, use_fp8=use_fp8, use_nvfp4=use_nvfp4, recv_x=recv_x,
                                    recv_scales=recv_scales), None, None, handle
    if num_experts is None:
        raise ValueError("num_experts is required with topk_idx")
    _need(topk_idx, "topk_idx", (torch.int64, torch.int32), ndim=2)
    T, k = topk_idx.shape
    dev = topk_idx.device
    if handle is None:
        handle = EPHandle(T, k, num_experts, num_segments, expert_alignment, max_recv_rows, device=dev)
    elif (handle.num_tokens, handle.num_topk, handle.num_experts) != (T, k, num_experts):
        raise ValueError("handle shape does not match topk_idx / num_experts")
    if topk_weights is not None:
        _need(topk_weights, "topk_weights", (torch.float32,), dev, 2)
        if tuple(topk_weights.shape) != (T, k):
            raise ValueError("topk_weights must have the shape of topk_idx")
    R = handle.max_recv_rows
    ri = torch.empty(R, dtype=torch.int32, device=dev) if recv_topk_idx is None else recv_topk_idx
    rw = torch.empty(R, dtype=torch.float32, device=dev) if recv_topk_weights is None else recv_topk_weights
    _need(ri, "recv_topk_idx", (torch.int32,), dev, 1)
    _need(rw, "recv_topk_weights", (torch.float32,), dev, 1)
    mode, x, x_scales, H, recv_x, recv_scales = _dispatch_args(x, handle, _bf16_mode(use_fp8, use_nvfp4),
                                                               recv_x, recv_scales)
    _check(lib().ep_layout_dispatch(handle.ref, topk_idx.data_ptr(), int(topk_idx.dtype == torch.int64),
                                    _ptr(topk_weights), ri.data_ptr(), rw.data_ptr(),
                                    handle.workspace_ptr, handle.workspace_bytes, mode, x.data_ptr(),
                                    _ptr(x_scales), H, recv_x.data_ptr(), _ptr(recv_scales),
                                    _stream(dev)), "dispatch")
    out = recv_x if mode == EP_X_BF16 else (recv_x, recv_scales)
    return out, ri, rw, handle


def combine(y: torch.Tensor, handle: EPHandle, topk_weights: Optional[torch.Tensor] = None, *,
            recv_topk_weights: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None):
    """MoE combine -> (out bf16 [T,H], combined weights [T,k] or None).

    topk_weights [T,k] f32 weights the sum (combine_forward); None sums the k
    rows unweighted (dispatch_backward).  recv_topk_weights [max_recv_rows]
    (e.g. the gradient of recv_topk_weights) is gathered back to [T,k]."""
    dev = handle.device
    _need(y, "y", (torch.bfloat16,), dev, 2)
    if y.shape[0] != handle.max_recv_rows:
        raise ValueError("y must have max_recv_rows rows")
    T, k, H = handle.num_tokens, handle.num_topk, y.shape[1]
    if topk_weights is not None:
        _need(topk_weights, "topk_weights", (torch.float32,), dev, 2)
        if tuple(topk_weights.shape) != (T, k):
            raise ValueError("topk_weights must be [T, k]")
    out_w = None
    if recv_topk_weights is not None:
        _need(recv_topk_weights, "recv_topk_weights", (torch.float32,), dev, 1)
        if recv_topk_weights.shape[0] != handle.max_recv_rows:
            raise ValueError("recv_topk_weights must have max_recv_rows entries")
        out_w = torch.empty(T, k, dtype=torch.float32, device=dev)
    if out is None:
        out = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
    _need(out, "out", (torch.bfloat16,), dev, 2)
    _check(lib().ep_combine(handle.ref, y.data_ptr(), H, _ptr(topk_weights), _ptr(recv_topk_weights),
                            _ptr(out_w), out.data_ptr(), _stream(dev)), "combine")
    return out, out_w


def combine_fp8(y_q: torch.Tensor, y_scales: torch.Tensor, handle: EPHandle,
                topk_weights: Optional[torch.Tensor] = None, *, out: Optional[torch.Tensor] = None):
    """Combine of FP8 expert outputs: y_q [max_recv_rows, H] e4m3 (or uint8)
    codes with y_scales [max_recv_rows, H/128] f32, in the layout of the FP8
    dispatch's output.  Each value is decode(q) * scale (binary32), summed
    like combine.  -> out [T, H] bf16."""
    dev = handle.device
    _need(y_q, "y_q", (torch.float8_e4m3fn, torch.uint8), dev, 2)
    _need(y_scales, "y_scales", (torch.float32,), dev, 2)
    rows, H = y_q.shape
    if rows != handle.max_recv_rows or tuple(y_scales.shape) != (rows, H // 128):
        raise ValueError("y_q must be [max_recv_rows, hidden] and y_scales [max_recv_rows, hidden/128]")
    if topk_weights is not None:
        _need(topk_weights, "topk_weights", (torch.float32,), dev, 2)
    if out is None:
        out = torch.empty(handle.num_tokens, H, dtype=torch.bfloat16, device=dev)
    _need(out, "out", (torch.bfloat16,), dev, 2)
    _check(lib().ep_combine_fp8(handle.ref, y_q.data_ptr(), y_scales.data_ptr(), H, _ptr(topk_weights),
                                out.data_ptr(), _stream(dev)), "combine_fp8")
    return out


def combine_backward(grad_out: torch.Tensor, y: torch.Tensor, handle: EPHandle,
                     topk_weights: Optional[torch.Tensor] = None, *,
                     grad_y: Optional[torch.Tensor] = None,
                     grad_weights: Optional[torch.Tensor] = None):
    """Backward of combine(y, handle, topk_weights) for the output gradient
    grad_out [T,H] bf16 -> (grad_y [max_recv_rows,H] bf16, grad_weights [T,k] f32)."""
    dev = handle.device
    T, k = handle.num_tokens, handle.num_topk
    _need(grad_out, "grad_out", (torch.bfloat16,), dev, 2)
    _need(y, "y", (torch.bfloat16,), dev, 2)
    H = grad_out.shape[1]
    if tuple(grad_out.shape) != (T, H) or tuple(y.shape) != (handle.max_recv_rows, H):
        raise ValueError("grad_out must be [T, hidden] and y [max_recv_rows, hidden]")
    if topk_weights is not None:
        _need(topk_weights, "topk_weights", (torch.float32,), dev, 2)
        if tuple(topk_weights.shape) != (T, k):
            raise ValueError("topk_weights must be [T, k]")
    if grad_y is None:
        grad_y = torch.empty_like(y)
    if grad_weights is None:
        grad_weights = torch.empty(T, k, dtype=torch.float32, device=dev)
    _need(grad_y, "grad_y", (torch.bfloat16,), dev, 2)
    _need(grad_weights, "grad_weights", (torch.float32,), dev, 2)
    _check(lib().ep_combine_backward(handle.ref, grad_out.data_ptr(), y.data_ptr(), H, _ptr(topk_weights),
                                     grad_y.data_ptr(), grad_weights.data_ptr(), _stream(dev)),
           "combine_backward")
    return grad_y, grad_weights


def dispatch_mn_scales(x: XType, handle: EPHandle, *, recv_x: Optional[torch.Tensor] = None,
                       recv_scales_mn: Optional[torch.Tensor] = None, scales_ld: Optional[int] = None):
    """FP8 dispatch with GEMM-ready scales: recv_scales_mn [H/128, scales_ld]
    (MN-major, scales_ld = max_recv_rows rounded up to 4 by default).
    x is bf16 (quantised here) or an (x_fp8, scales) tuple."""
    dev = handle.device
    rows = handle.max_recv_rows
    if scales_ld is None:
        scales_ld = (rows + 3) // 4 * 4
    xt = x[0] if isinstance(x, (tuple, list)) else x
    H = xt.shape[1]
    if recv_scales_mn is None:
        recv_scales_mn = torch.empty(H // 128, scales_ld, dtype=torch.float32, device=dev)
    _need(recv_scales_mn, "recv_scales_mn", (torch.float32,), dev, 2)
    if tuple(recv_scales_mn.shape) != (H // 128, scales_ld):
        raise ValueError("recv_scales_mn must be [hidden/128, scales_ld]")
    mode, x, x_scales, H, recv_x, _ = _dispatch_args(x, handle, EP_X_BF16_TO_FP8, recv_x, None, row_scales=False)
    _check(lib().ep_dispatch_mn_scales(handle.ref, mode, x.data_ptr(), _ptr(x_scales), H, recv_x.data_ptr(),
                                       recv_scales_mn.data_ptr(), scales_ld, _stream(dev)), "dispatch_mn_scales")
    return recv_x, recv_scales_mn
