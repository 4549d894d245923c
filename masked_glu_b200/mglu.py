"""Thin ctypes binding of libmglu.so (see include/mglu.h).

Argument marshalling only: tensors are passed as raw device pointers with the
current torch stream; every step of the computation runs in the library's
CUDA kernels.  There is no fallback: if the library is missing, or a call
fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmglu.so")
HEADER = os.path.join(os.path.dirname(_PKG), "include", "mglu.h")

OK, ERR_INVALID, ERR_UNSUPPORTED, ERR_ALIGN, ERR_CUDA, ERR_TIMEOUT = 0, -1, -2, -3, -4, -5
ACTS = {"swish": 0, "gelu": 1, "relu": 2}
GATE_DENSE = 16  # OR-ed into act: the dense-gate ablation (act names may end in "+dense_gate")
DTYPES = {torch.bfloat16: 0, torch.float32: 1}
PATH_DECODE, PATH_PREFILL, PATH_F32 = 0, 1, 2

_lib = None


class MGLUError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = f"{where}: {status_string(status)} ({status})"
        if status == ERR_CUDA:
            msg += f": {last_cuda_error()}"
        super().__init__(msg)


def header_functions():
    """Names of the functions include/mglu.h declares."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*(mglu_[a-z_0-9]+)\s*\(", text, flags=re.M)


def lib() -> ctypes.CDLL:
    """Load libmglu.so (built in-tree by ``python -m masked_glu_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m masked_glu_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I64, I32, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
        sig = {
            "mglu_packed_bytes": (SZ, [I32, I64, I64]),
            "mglu_pack_masks": (I32, [P, I32, I64, I64, P, P]),
            "mglu_unpack_masks": (I32, [P, I32, I64, I64, P, P]),
            "mglu_pack_mask_logits": (I32, [P, I32, I64, I64, P, P]),
            "mglu_scratch_bytes": (SZ, [I64]),
            "mglu_forward": (I32, [P, I64, I64, P, I64, P, I32, I32, I32, P, P, SZ, P]),
            "mglu_down_proj": (I32, [P, I64, I64, P, I64, I32, P, P, SZ, P]),
            "mglu_route_topk": (I32, [P, I64, I64, P, I32, I32, I32, I32, P, P, P]),
            "mglu_forward_weighted": (I32, [P, I64, I64, P, I64, P, I32, I32, I32, P, P, P, SZ, P]),
            "mglu_forward_partials": (I32, [P, I64, I64, P, I64, P, I32, P, P, SZ, P]),
            "mglu_forward_routed": (I32, [P, I64, I64, P, I64, P, I32, P, I32, I32, I32, I32, P, P, P, P, SZ, P]),
            "mglu_workspace_bytes": (SZ, [I64, I64, I64, I32, I32]),
            "mglu_forward_down": (I32, [P, I64, I64, P, I64, P, I32, I32, I32, P, P, SZ, P, P]),
            "mglu_forward_decode_static": (I32, [P, I64, I64, P, I64, P, I32, I32, P, P]),
            "mglu_host_workspace_bytes": (SZ, [I64, I64, I64, I32, I32, I32]),
            "mglu_backward_workspace_bytes": (SZ, [I64, I64, I64, I32]),
            "mglu_backward": (I32, [P, I64, I64, P, I64, P, I32, I32, P, P, P, P, P, SZ, P]),
            "mglu_forward_host": (I32, [P, I64, I64, P, I64, P, I32, I32, I32, P, P, SZ, P, P]),
            "mglu_forward_path": (I32, [I64, I32]),
            "mglu_set_decode_max_tokens": (I32, [I32]),
            "mglu_last_device_status": (I32, [P]),
            "mglu_last_cuda_error": (ctypes.c_char_p, []),
            "mglu_status_string": (ctypes.c_char_p, [I32]),
            "mglu_kernel_launches": (ctypes.c_uint64, []),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().mglu_status_string(int(status)).decode()


def last_cuda_error() -> str:
    return lib().mglu_last_cuda_error().decode()


def _check(rc: int, where: str) -> None:
    if rc != OK:
        raise MGLUError(rc, where)


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not (t.is_cuda and t.is_contiguous()):
        raise ValueError("tensors must be contiguous and on a CUDA device")
    return t.data_ptr()


def _hptr(t: torch.Tensor) -> int:
    if t.is_cuda or not t.is_contiguous():
        raise ValueError("host tensors must be contiguous CPU tensors")
    return t.data_ptr()


def _dtype(t: torch.Tensor) -> int:
    if t.dtype not in DTYPES:
        raise ValueError(f"unsupported dtype {t.dtype}")
    return DTYPES[t.dtype]


def _act(act) -> int:
    if isinstance(act, str):
        name, _, flag = act.partition("+")
        if flag not in ("", "dense_gate"):
            raise ValueError(f"unknown act modifier {flag!r}")
        return ACTS[name] | (GATE_DENSE if flag else 0)
    return int(act)


def packed_bytes(n_m: int, d: int, h: int) -> int:
    return int(lib().mglu_packed_bytes(n_m, d, h))


def pack_masks(masks: torch.Tensor, stream=None) -> torch.Tensor:
    """masks [n_m][h][d] uint8 (0/1) on the GPU -> packed uint8 stream."""
    n_m, h, d = masks.shape
    out = torch.empty(packed_bytes(n_m, d, h), dtype=torch.uint8, device=masks.device)
    _check(lib().mglu_pack_masks(_ptr(masks), n_m, d, h, _ptr(out), _stream(stream)), "mglu_pack_masks")
    return out


def pack_mask_logits(logits: torch.Tensor, stream=None) -> torch.Tensor:
    """logits [n_m][h][d] float16 on the GPU -> packed stream of the masks
    logit > 0."""
    if logits.dtype != torch.float16:
        raise ValueError("mask logits must be float16")
    n_m, h, d = logits.shape
    out = torch.empty(packed_bytes(n_m, d, h), dtype=torch.uint8, device=logits.device)
    _check(lib().mglu_pack_mask_logits(_ptr(logits), n_m, d, h, _ptr(out), _stream(stream)), "mglu_pack_mask_logits")
    return out


def unpack_masks(packed: torch.Tensor, n_m: int, d: int, h: int, stream=None) -> torch.Tensor:
    out = torch.empty((n_m, h, d), dtype=torch.uint8, device=packed.device)
    _check(lib().mglu_unpack_masks(_ptr(packed), n_m, d, h, _ptr(out), _stream(stream)), "mglu_unpack_masks")
    return out


def scratch_bytes(rows: int) -> int:
    return int(lib().mglu_scratch_bytes(rows))


_scratch = {}


def default_scratch(rows: int, device) -> torch.Tensor:
    """A zero-filled scratch buffer per device, grown on demand and shared by
    calls that pass none.  Calls on several streams at once must pass their
    own buffers (the decode kernel's partial slots are not safe to share)."""
    dev = torch.device(device)
    key = dev.index if dev.index is not None else torch.cuda.current_device()
    need = scratch_bytes(rows)
    buf = _scratch.get(key)
    if buf is None or buf.numel() < need:
        buf = torch.zeros(need, dtype=torch.uint8, device=dev)
        _scratch[key] = buf
    return buf


def _nbytes(t: Optional[torch.Tensor]) -> int:
    return 0 if t is None else t.numel() * t.element_size()


def forward(x: torch.Tensor, W: torch.Tensor, packed: torch.Tensor, n_m: int, act="swish",
            out: Optional[torch.Tensor] = None, scratch: Optional[torch.Tensor] = None,
            stream=None) -> torch.Tensor:
    """out [T][h] = MGLU(x [T][d]) with W [h][d] and packed masks."""
    T, d = x.shape
    h = W.shape[0]
    if W.shape[1] != d or W.dtype != x.dtype:
        raise ValueError("W must be [h][d] with x's dtype")
    if out is None:
        out = torch.empty((T, h), dtype=x.dtype, device=x.device)
    if scratch is None:
        scratch = default_scratch(h, x.device)
    _check(lib().mglu_forward(_ptr(x), T, d, _ptr(W), h, _ptr(packed), n_m, _act(act), _dtype(x),
                              _ptr(out), _ptr(scratch), _nbytes(scratch), _stream(stream)), "mglu_forward")
    return out


ROUTE_MODES = {"hard": 0, "softmax": 1}


def route_topk(x: torch.Tensor, W_r: torch.Tensor, k: int, mode="hard", weights: Optional[torch.Tensor] = None,
               scores: Optional[torch.Tensor] = None, stream=None):
    """Router scores x W_r^T, top-k per token, mask weights [T][n_m] float.
    Returns (weights, scores)."""
    T, d = x.shape
    n_m = W_r.shape[0]
    if W_r.shape[1] != d or W_r.dtype != x.dtype:
        raise ValueError("W_r must be [n_m][d] with x's dtype")
    if weights is None:
        weights = torch.empty((T, n_m), dtype=torch.float32, device=x.device)
    if scores is None:
        scores = torch.empty((T, n_m), dtype=torch.float32, device=x.device)
    _check(lib().mglu_route_topk(_ptr(x), T, d, _ptr(W_r), n_m, int(k), ROUTE_MODES.get(mode, mode), _dtype(x),
                                 _ptr(weights), _ptr(scores), _stream(stream)), "mglu_route_topk")
    return weights, scores


def forward_weighted(x: torch.Tensor, W: torch.Tensor, packed: torch.Tensor, n_m: int, mask_weights: torch.Tensor,
                     act="swish", out: Optional[torch.Tensor] = None, scratch: Optional[torch.Tensor] = None,
                     stream=None) -> torch.Tensor:
    """out [T][h] = sum_i w[b, i] act(g_i) v_i with mask_weights [T][n_m] float."""
    T, d = x.shape
    h = W.shape[0]
    if W.shape[1] != d or W.dtype != x.dtype:
        raise ValueError("W must be [h][d] with x's dtype")
    if mask_weights.shape != (T, n_m) or mask_weights.dtype != torch.float32:
        raise ValueError("mask_weights must be [T][n_m] float32")
    if out is None:
        out = torch.empty((T, h), dtype=x.dtype, device=x.device)
    if scratch is None:
        scratch = default_scratch(h, x.device)
    _check(lib().mglu_forward_weighted(_ptr(x), T, d, _ptr(W), h, _ptr(packed), n_m, _act(act), _dtype(x),
                                       _ptr(mask_weights), _ptr(out), _ptr(scratch), _nbytes(scratch),
                                       _stream(stream)), "mglu_forward_weighted")
    return out


def forward_routed(x: torch.Tensor, W: torch.Tensor, packed: torch.Tensor, n_m: int, W_r: torch.Tensor, k: int,
                   mode="hard", act="swish", out: Optional[torch.Tensor] = None,
                   weights: Optional[torch.Tensor] = None, scores: Optional[torch.Tensor] = None,
                   scratch: Optional[torch.Tensor] = None, stream=None):
    """route_topk then forward_weighted in one call (on the decode kernel the
    router runs inside the forward kernel).  Returns (out, weights, scores)."""
    T, d = x.shape
    h = W.shape[0]
    if W.shape[1] != d or W.dtype != x.dtype:
        raise ValueError("W must be [h][d] with x's dtype")
    if W_r.shape != (n_m, d) or W_r.dtype != x.dtype:
        raise ValueError("W_r must be [n_m][d] with x's dtype")
    if out is None:
        out = torch.empty((T, h), dtype=x.dtype, device=x.device)
    if weights is None:
        weights = torch.empty((T, n_m), dtype=torch.float32, device=x.device)
    if scores is None:
        scores = torch.empty((T, n_m), dtype=torch.float32, device=x.device)
    if scratch is None:
        scratch = default_scratch(h, x.device)
    _check(lib().mglu_forward_routed(_ptr(x), T, d, _ptr(W), h, _ptr(packed), n_m, _ptr(W_r), int(k),
                                     ROUTE_MODES.get(mode, mode), _act(act), _dtype(x), _ptr(weights), _ptr(scores),
                                     _ptr(out), _ptr(scratch), _nbytes(scratch), _stream(stream)),
           "mglu_forward_routed")
    return out, weights, scores


def forward_partials(x: torch.Tensor, W: torch.Tensor, packed: torch.Tensor, n_m: int,
                     scratch: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """The decode kernel's unrounded partial sums, float32 [2 n_m + 1][T][h]:
    plane 0 = D = x W^T, plane 1 + 2i = g_i, plane 2 + 2i = v_i (bf16, T <= 16)."""
    T, d = x.shape
    h = W.shape[0]
    if W.shape[1] != d or W.dtype != x.dtype:
        raise ValueError("W must be [h][d] with x's dtype")
    out = torch.empty((2 * n_m + 1, T, h), dtype=torch.float32, device=x.device)
    if scratch is None:
        scratch = default_scratch(h, x.device)
    _check(lib().mglu_forward_partials(_ptr(x), T, d, _ptr(W), h, _ptr(packed), n_m, _ptr(out), _ptr(scratch),
                                       _nbytes(scratch), _stream(stream)), "mglu_forward_partials")
    return out


def forward_decode_static(x: torch.Tensor, W: torch.Tensor, packed: torch.Tensor, n_m: int, act="swish",
                          out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """mglu_forward on the decode kernel (bf16, T <= 16) using the library's
    built-in scratch instead of a caller buffer."""
    T, d = x.shape
    h = W.shape[0]
    if W.shape[1] != d or W.dtype != x.dtype:
        raise ValueError("W must be [h][d] with x's dtype")
    if out is None:
        out = torch.empty((T, h), dtype=x.dtype, device=x.device)
    _check(lib().mglu_forward_decode_static(_ptr(x), T, d, _ptr(W), h, _ptr(packed), n_m, _act(act), _ptr(out),
                                            _stream(stream)), "mglu_forward_decode_static")
    return out


def down_proj(hid: torch.Tensor, W_down: torch.Tensor, out: Optional[torch.Tensor] = None,
              scratch: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """y [T][d] = hid [T][h] @ W_down[d][h]^T."""
    T, h = hid.shape
    d = W_down.shape[0]
    if out is None:
        out = torch.empty((T, d), dtype=hid.dtype, device=hid.device)
    if scratch is None:
        scratch = default_scratch(d, hid.device)
    _check(lib().mglu_down_proj(_ptr(hid), T, h, _ptr(W_down), d, _dtype(hid), _ptr(out), _ptr(scratch),
                                _nbytes(scratch), _stream(stream)), "mglu_down_proj")
    return out


def workspace_bytes(T: int, d: int, h: int, n_m: int, dtype=torch.bfloat16) -> int:
    return int(lib().mglu_workspace_bytes(T, d, h, n_m, DTYPES[dtype]))


def forward_down(x: torch.Tensor, W: torch.Tensor, packed: torch.Tensor, n_m: int, W_down: torch.Tensor,
                 act="swish", workspace: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                 stream=None) -> torch.Tensor:
    """y = MGLU(x) @ W_down^T through a caller-owned workspace."""
    T, d = x.shape
    h = W.shape[0]
    need = workspace_bytes(T, d, h, n_m, x.dtype)
    if workspace is None:
        workspace = torch.zeros(max(need, 256), dtype=torch.uint8, device=x.device)
    if out is None:
        out = torch.empty((T, d), dtype=x.dtype, device=x.device)
    _check(lib().mglu_forward_down(_ptr(x), T, d, _ptr(W), h, _ptr(packed), n_m, _act(act), _dtype(x),
                                   _ptr(W_down), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                   _ptr(out), _stream(stream)), "mglu_forward_down")
    return out


def host_workspace_bytes(T: int, d: int, h: int, n_m: int, dtype=torch.bfloat16, with_down=False) -> int:
    return int(lib().mglu_host_workspace_bytes(T, d, h, n_m, DTYPES[dtype], 1 if with_down else 0))


def forward_host(x_host: torch.Tensor, W: torch.Tensor, packed: torch.Tensor, n_m: int, act="swish",
                 W_down: Optional[torch.Tensor] = None, out_host: Optional[torch.Tensor] = None,
                 workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """The forward (or, with W_down, the FFN block) on host activations: one
    library call copies x_host to the device, runs the kernels and copies the
    result into out_host, in order on the stream.  Pin the host tensors for
    asynchronous copies; out_host is valid after the stream synchronizes."""
    T, d = x_host.shape
    h = W.shape[0]
    if x_host.is_cuda or (out_host is not None and out_host.is_cuda):
        raise ValueError("x_host and out_host must be host tensors")
    if out_host is None:
        out_host = torch.empty((T, d if W_down is not None else h), dtype=x_host.dtype, pin_memory=True)
    need = host_workspace_bytes(T, d, h, n_m, x_host.dtype, W_down is not None)
    if workspace is None:
        workspace = torch.zeros(max(need, 256), dtype=torch.uint8, device=W.device)
    _check(lib().mglu_forward_host(_hptr(x_host), T, d, _ptr(W), h, _ptr(packed), n_m, _act(act), _dtype(x_host),
                                   _ptr(W_down), _ptr(workspace), _nbytes(workspace), _hptr(out_host),
                                   _stream(stream)), "mglu_forward_host")
    return out_host


def backward(x: torch.Tensor, W: torch.Tensor, packed: torch.Tensor, n_m: int, dout: torch.Tensor, act="swish",
             with_logits: bool = True, workspace: Optional[torch.Tensor] = None, stream=None):
    """Gradients (dx [T][d], dW [h][d], dlogits [n_m][h][d] or None) of L
    through out = MGLU(x) for dout = dL/dout [T][h], float32."""
    T, d = x.shape
    h = W.shape[0]
    if dout.shape != (T, h) or dout.dtype != x.dtype:
        raise ValueError("dout must be [T][h] with x's dtype")
    dx = torch.empty((T, d), dtype=torch.float32, device=x.device)
    dW = torch.empty((h, d), dtype=torch.float32, device=x.device)
    dM = torch.empty((n_m, h, d), dtype=torch.float32, device=x.device) if with_logits else None
    need = int(lib().mglu_backward_workspace_bytes(T, d, h, n_m))
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=x.device)
    _check(lib().mglu_backward(_ptr(x), T, d, _ptr(W), h, _ptr(packed), n_m, _act(act), _ptr(dout), _ptr(dx),
                               _ptr(dW), _ptr(dM), _ptr(workspace), _nbytes(workspace), _stream(stream)),
           "mglu_backward")
    return dx, dW, dM


def forward_path(T: int, dtype=torch.bfloat16) -> int:
    return int(lib().mglu_forward_path(T, DTYPES[dtype]))


def set_decode_max_tokens(t: int) -> int:
    prev = lib().mglu_set_decode_max_tokens(int(t))
    if prev < 0:
        raise MGLUError(prev, "mglu_set_decode_max_tokens")
    return prev


def last_device_status(stream=None) -> int:
    return int(lib().mglu_last_device_status(_stream(stream)))


def kernel_launches() -> int:
    """Kernels the library has launched in this process so far."""
    return int(lib().mglu_kernel_launches())
