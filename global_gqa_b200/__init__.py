"""Python binding of libg3attn (Gemma 3 5:1 block attention on B200).

Argument marshalling only: every step of the computation runs in the CUDA
library behind the C ABI declared in include/g3attn.h.  torch supplies device
memory and the current stream.  There is no fallback: if the library is not
built or no CUDA device is present, the calls raise.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional, Tuple

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB_PATH = os.path.join(HERE, "libg3attn.so")
HEADER_PATH = os.path.join(ROOT, "include", "g3attn.h")

LOCAL = 0
GLOBAL = 1

STATUS = {0: "G3_OK", 1: "G3_ERR_INVALID_ARG", 2: "G3_ERR_UNSUPPORTED", 3: "G3_ERR_WORKSPACE",
          4: "G3_ERR_CUDA", 5: "G3_ERR_TIMEOUT"}


class G3Error(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}: {detail}")


class KernelTrace(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 48), ("launches", ctypes.c_int64), ("total_ms", ctypes.c_double)]


_lib = None

_vp, _i32, _f32, _sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t

_SIGS = {
    "g3attn_prefill_workspace_size": (_sz, [_i32] * 5),
    "g3attn_prefill": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_int, _i32, _f32, _f32, _vp, _i32,
                                      _i32, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _i32, _vp, _sz, _vp]),
    "g3attn_prefill_chunk_workspace_size": (_sz, [_i32] * 6 + [ctypes.c_int, _i32]),
    "g3attn_prefill_chunk": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, ctypes.c_int, _i32,
                                            _f32, _f32, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _vp,
                                            _sz, _vp]),
    "g3attn_prefill_backward_workspace_size": (_sz, [_i32] * 5),
    "g3attn_prefill_backward": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_int, _i32, _f32, _f32, _vp,
                                               _i32, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _vp,
                                               _vp, _vp, _vp, _sz, _vp]),
    "g3attn_soft_tokens": (ctypes.c_int, [_vp, _vp, _i32, _i32, _i32, _i32, _i32, _vp, _vp]),
    "g3attn_decode_workspace_size": (_sz, [_i32] * 5),
    "g3attn_decode": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _i32, ctypes.c_int, _i32,
                                     _f32, _f32, _i32, _i32, _i32, _i32, _vp, _vp, _sz, _vp]),
    "g3attn_decode_no_alloc": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _i32, ctypes.c_int,
                                              _i32, _f32, _f32, _i32, _i32, _i32, _i32, _vp, _vp]),
    "g3attn_check_device_error": (ctypes.c_int, [_vp, _vp]),
    "g3attn_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "g3attn_last_error": (ctypes.c_char_p, []),
    "g3attn_trace_enable": (ctypes.c_int, [ctypes.c_int]),
    "g3attn_trace_collect": (_i32, [ctypes.POINTER(KernelTrace), _i32]),
}


def lib() -> ctypes.CDLL:
    """The loaded C library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m global_gqa_b200.build`")
        h = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(h, name)
            fn.restype = res
            fn.argtypes = args
        _lib = h
    return _lib


def header_functions() -> list:
    """Names of the functions include/g3attn.h declares."""
    with open(HEADER_PATH) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(g3attn_\w+)\s*\(", text)))


def _check(status: int, where: str) -> None:
    if status != 0:
        detail = lib().g3attn_last_error().decode(errors="replace")
        raise G3Error(status, where, detail)


def prefill_workspace_size(B: int, S: int, Hq: int, Hkv: int, D: int) -> int:
    return int(lib().g3attn_prefill_workspace_size(B, S, Hq, Hkv, D))


def prefill_chunk_workspace_size(B: int, C: int, Hq: int, Hkv: int, D: int, start: int, layer_kind: int,
                                 window: int) -> int:
    return int(lib().g3attn_prefill_chunk_workspace_size(B, C, Hq, Hkv, D, start, int(layer_kind), window))


def prefill_backward_workspace_size(B: int, S: int, Hq: int, Hkv: int, D: int) -> int:
    return int(lib().g3attn_prefill_backward_workspace_size(B, S, Hq, Hkv, D))


def decode_workspace_size(B: int, Hq: int, Hkv: int, D: int, max_seq_len: int) -> int:
    return int(lib().g3attn_decode_workspace_size(B, Hq, Hkv, D, max_seq_len))


# ----------------------------------------------------------- torch plumbing
def _torch():
    import torch
    return torch


_workspaces = {}


def workspace(nbytes: int, device, tag: str = "default", stream=None):
    """A cached uint8 device buffer of at least nbytes (256-byte aligned).

    One buffer per (device, tag, stream): calls on one stream run in order and
    may share it, calls on different streams may overlap and must not (stream
    None is the device's current stream, as in the calls).
    """
    torch = _torch()
    device = torch.device(device)
    if device.index is None:  # "cuda" means the current device: name it as tensors do
        device = torch.device("cuda", torch.cuda.current_device())
    s = stream if stream is not None else torch.cuda.current_stream(device)
    key = (str(device), tag, int(s.cuda_stream))
    buf = _workspaces.get(key)
    if buf is None or buf.numel() < nbytes:
        # Allocated on the stream that uses it, so that when a larger buffer
        # replaces it, torch reuses the old memory only after that stream's
        # earlier calls have finished with it.
        with torch.cuda.stream(s):
            buf = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
        _workspaces[key] = buf
    return buf


def release_workspaces(device=None, stream=None) -> int:
    """Drops the cached workspaces (all of them, or those of one device and/or
    stream) so torch can reuse their memory; returns how many were dropped.
    A server that makes a stream per request calls this when the stream is
    retired.  Work already queued keeps its buffer alive through torch's
    stream-ordered allocator."""
    torch = _torch()
    dev = None
    if device is not None:
        dev = torch.device(device)
        if dev.index is None:
            dev = torch.device("cuda", torch.cuda.current_device())
    sid = None if stream is None else int(stream.cuda_stream)
    drop = [k for k in _workspaces if (dev is None or k[0] == str(dev)) and (sid is None or k[2] == sid)]
    for k in drop:
        del _workspaces[k]
    return len(drop)


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream_ptr(stream, device) -> int:
    torch = _torch()
    if stream is None:
        return torch.cuda.current_stream(device).cuda_stream
    if stream.device != device:
        raise ValueError(f"stream belongs to {stream.device}; the call runs on {device}")
    return stream.cuda_stream


def _on_device(device, **tensors) -> None:
    """Every tensor of one call lives on the GPU the call runs on (the library
    launches on the current device, which the entry points set to it)."""
    for name, t in tensors.items():
        if t is not None and t.device != device:
            raise ValueError(f"{name} is on {t.device}; every tensor of the call must be on {device}")


def _ws(ws, nbytes: int, device, tag: str = "default", stream=None):
    """The caller's workspace (checked) or the stream's cached one, with its size in bytes."""
    torch = _torch()
    if ws is None:
        ws = workspace(nbytes, device, tag, stream)
    elif not isinstance(ws, torch.Tensor) or ws.device != device or not ws.is_contiguous():
        raise ValueError(f"ws must be a contiguous tensor on {device}")
    return ws, ws.numel() * ws.element_size()


def _req(t, name, dtype, shape=None):
    torch = _torch()
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be on a CUDA device (no CPU path exists)")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def prefill(q, k, v, q_gamma, k_gamma, positions, layer_kind: int, window: int, rope_base: float,
            interp_factor: float, image_spans=None, *, out=None, return_lse: bool = False,
            k_cache=None, v_cache=None, ws=None, stream=None):
    """One attention layer over full sequences; returns out (and lse).

    q [B,S,Hq,D] bf16, k/v [B,S,Hkv,D] bf16 (raw projections), gammas fp32
    [D], positions int32 [B,S], image_spans int32 [B,n,2] or None.
    """
    torch = _torch()
    _req(q, "q", torch.bfloat16)
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    _req(k, "k", torch.bfloat16, (B, S, Hkv, D))
    _req(v, "v", torch.bfloat16, (B, S, Hkv, D))
    _req(q_gamma, "q_gamma", torch.float32, (D,))
    _req(k_gamma, "k_gamma", torch.float32, (D,))
    _req(positions, "positions", torch.int32, (B, S))
    n_spans = 0
    if image_spans is not None:
        _req(image_spans, "image_spans", torch.int32)
        if image_spans.dim() != 3 or image_spans.shape[0] != B or image_spans.shape[2] != 2:
            raise ValueError("image_spans must be [B, n, 2]")
        n_spans = int(image_spans.shape[1])
        if n_spans == 0:
            image_spans = None
    if out is None:
        out = torch.empty_like(q)
    _req(out, "out", torch.bfloat16, (B, S, Hq, D))
    lse = torch.empty(B, Hq, S, dtype=torch.float32, device=q.device) if return_lse else None
    cap = 0
    if k_cache is not None:
        _req(k_cache, "k_cache", torch.bfloat16)
        if k_cache.dim() != 4 or k_cache.shape[0] != B or k_cache.shape[1] != Hkv or k_cache.shape[3] != D:
            raise ValueError("k_cache must be [B, Hkv, capacity, D]")
        _req(v_cache, "v_cache", torch.bfloat16, tuple(k_cache.shape))
        cap = int(k_cache.shape[2])
    dev = q.device
    _on_device(dev, k=k, v=v, q_gamma=q_gamma, k_gamma=k_gamma, positions=positions, image_spans=image_spans,
               out=out, k_cache=k_cache, v_cache=v_cache)
    wsb, ws_bytes = _ws(ws, prefill_workspace_size(B, S, Hq, Hkv, D), dev, stream=stream)
    with torch.cuda.device(dev):
        st = lib().g3attn_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(q_gamma), _ptr(k_gamma), _ptr(positions),
                                  int(layer_kind), int(window), float(rope_base), float(interp_factor),
                                  _ptr(image_spans), n_spans, B, S, Hq, Hkv, D, _ptr(out), _ptr(lse),
                                  _ptr(k_cache), _ptr(v_cache), cap, wsb.data_ptr(), ws_bytes,
                                  _stream_ptr(stream, dev))
    _check(st, "g3attn_prefill")
    return (out, lse) if return_lse else out


def prefill_backward(q, k, v, q_gamma, k_gamma, positions, layer_kind: int, window: int, rope_base: float,
                     interp_factor: float, image_spans, out, lse, dout, *, grads=None, ws=None, stream=None):
    """Gradients of one prefill layer: returns dict(dq, dk, dv, dq_gamma, dk_gamma).

    Arguments as for prefill, plus the forward's out [B,S,Hq,D] bf16 and lse
    [B,Hq,S] fp32 and the output gradient dout [B,S,Hq,D] bf16.  `grads` may
    hold preallocated outputs under the same keys.
    """
    torch = _torch()
    _req(q, "q", torch.bfloat16)
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    _req(k, "k", torch.bfloat16, (B, S, Hkv, D))
    _req(v, "v", torch.bfloat16, (B, S, Hkv, D))
    _req(q_gamma, "q_gamma", torch.float32, (D,))
    _req(k_gamma, "k_gamma", torch.float32, (D,))
    _req(positions, "positions", torch.int32, (B, S))
    _req(out, "out", torch.bfloat16, (B, S, Hq, D))
    _req(lse, "lse", torch.float32, (B, Hq, S))
    _req(dout, "dout", torch.bfloat16, (B, S, Hq, D))
    n_spans = 0
    if image_spans is not None:
        _req(image_spans, "image_spans", torch.int32)
        if image_spans.dim() != 3 or image_spans.shape[0] != B or image_spans.shape[2] != 2:
            raise ValueError("image_spans must be [B, n, 2]")
        n_spans = int(image_spans.shape[1])
        if n_spans == 0:
            image_spans = None
    g = dict(grads) if grads is not None else {}
    g.setdefault("dq", torch.empty_like(q))
    g.setdefault("dk", torch.empty_like(k))
    g.setdefault("dv", torch.empty_like(v))
    g.setdefault("dq_gamma", torch.empty_like(q_gamma))
    g.setdefault("dk_gamma", torch.empty_like(k_gamma))
    _req(g["dq"], "dq", torch.bfloat16, (B, S, Hq, D))
    _req(g["dk"], "dk", torch.bfloat16, (B, S, Hkv, D))
    _req(g["dv"], "dv", torch.bfloat16, (B, S, Hkv, D))
    _req(g["dq_gamma"], "dq_gamma", torch.float32, (D,))
    _req(g["dk_gamma"], "dk_gamma", torch.float32, (D,))
    dev = q.device
    _on_device(dev, k=k, v=v, q_gamma=q_gamma, k_gamma=k_gamma, positions=positions, image_spans=image_spans,
               out=out, lse=lse, dout=dout, **g)
    wsb, ws_bytes = _ws(ws, prefill_backward_workspace_size(B, S, Hq, Hkv, D), dev, tag="backward",
                        stream=stream)
    with torch.cuda.device(dev):
        st = lib().g3attn_prefill_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(q_gamma), _ptr(k_gamma),
                                           _ptr(positions), int(layer_kind), int(window), float(rope_base),
                                           float(interp_factor), _ptr(image_spans), n_spans, B, S, Hq, Hkv, D,
                                           _ptr(out), _ptr(lse), _ptr(dout), _ptr(g["dq"]), _ptr(g["dk"]),
                                           _ptr(g["dv"]), _ptr(g["dq_gamma"]), _ptr(g["dk_gamma"]),
                                           wsb.data_ptr(), ws_bytes, _stream_ptr(stream, dev))
    _check(st, "g3attn_prefill_backward")
    return g


def decode(q, k_new, v_new, q_gamma, k_gamma, k_cache, v_cache, seq_lens, max_seq_len: int,
           layer_kind: int, window: int, rope_base: float, interp_factor: float, *, out=None,
           ws=None, stream=None):
    """One decode step: writes the new token into the cache and returns out [B,Hq,D]."""
    torch = _torch()
    _req(q, "q", torch.bfloat16)
    B, Hq, D = q.shape
    Hkv = k_new.shape[1]
    _req(k_new, "k_new", torch.bfloat16, (B, Hkv, D))
    _req(v_new, "v_new", torch.bfloat16, (B, Hkv, D))
    _req(q_gamma, "q_gamma", torch.float32, (D,))
    _req(k_gamma, "k_gamma", torch.float32, (D,))
    _req(k_cache, "k_cache", torch.bfloat16)
    cap = int(k_cache.shape[2])
    _req(k_cache, "k_cache", torch.bfloat16, (B, Hkv, cap, D))
    _req(v_cache, "v_cache", torch.bfloat16, (B, Hkv, cap, D))
    _req(seq_lens, "seq_lens", torch.int32, (B,))
    if out is None:
        out = torch.empty_like(q)
    _req(out, "out", torch.bfloat16, (B, Hq, D))
    dev = q.device
    _on_device(dev, k_new=k_new, v_new=v_new, q_gamma=q_gamma, k_gamma=k_gamma, k_cache=k_cache,
               v_cache=v_cache, seq_lens=seq_lens, out=out)
    # Decode keeps its own cached workspace: its launch clears the error word,
    # which would otherwise erase a prefill's unread device error.  A local
    # layer's query sees at most `window` ring slots, which bounds its scratch.
    visible = min(int(max_seq_len), int(window)) if layer_kind == LOCAL and window >= 1 else int(max_seq_len)
    wsb, ws_bytes = _ws(ws, decode_workspace_size(B, Hq, Hkv, D, visible), dev, tag="decode", stream=stream)
    with torch.cuda.device(dev):
        st = lib().g3attn_decode(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(q_gamma), _ptr(k_gamma),
                                 _ptr(k_cache), _ptr(v_cache), cap, _ptr(seq_lens), int(max_seq_len),
                                 int(layer_kind), int(window), float(rope_base), float(interp_factor),
                                 B, Hq, Hkv, D, _ptr(out), wsb.data_ptr(), ws_bytes, _stream_ptr(stream, dev))
    _check(st, "g3attn_decode")
    return out


def check_device_error(ws=None, device=None, stream=None) -> int:
    """Status recorded on the device by the last call using this workspace."""
    torch = _torch()
    if ws is None:
        dev = torch.device(device if device is not None else "cuda")
        ws = workspace(256, dev, stream=stream)
    if not isinstance(ws, torch.Tensor) or ws.device.type != "cuda":
        raise ValueError("ws must be a CUDA tensor")
    with torch.cuda.device(ws.device):
        return int(lib().g3attn_check_device_error(ws.data_ptr(), _stream_ptr(stream, ws.device)))


def trace_enable(on: bool = True) -> None:
    lib().g3attn_trace_enable(1 if on else 0)


def trace_collect() -> dict:
    arr = (KernelTrace * 32)()
    n = lib().g3attn_trace_collect(arr, 32)
    return {arr[i].name.decode(): (int(arr[i].launches), float(arr[i].total_ms)) for i in range(n)}


def prefill_chunk(q, k, v, q_gamma, k_gamma, positions, k_cache, v_cache, start: int, layer_kind: int,
                  window: int, rope_base: float, interp_factor: float, image_spans=None, *, out=None,
                  return_lse: bool = False, ws=None, stream=None):
    """The next C tokens of sequences whose first `start` tokens are cached; returns out (and lse).

    q [B,C,Hq,D] bf16, k/v [B,C,Hkv,D] bf16 (raw projections of the chunk),
    positions int32 [B,C], k_cache/v_cache bf16 [B,Hkv,cap,D] (updated in place),
    image_spans int32 [B,n,2] in whole-sequence token indices, or None.
    """
    torch = _torch()
    _req(q, "q", torch.bfloat16)
    B, C, Hq, D = q.shape
    Hkv = k.shape[2]
    _req(k, "k", torch.bfloat16, (B, C, Hkv, D))
    _req(v, "v", torch.bfloat16, (B, C, Hkv, D))
    _req(q_gamma, "q_gamma", torch.float32, (D,))
    _req(k_gamma, "k_gamma", torch.float32, (D,))
    _req(positions, "positions", torch.int32, (B, C))
    _req(k_cache, "k_cache", torch.bfloat16)
    _req(v_cache, "v_cache", torch.bfloat16, tuple(k_cache.shape))
    if k_cache.dim() != 4 or k_cache.shape[0] != B or k_cache.shape[1] != Hkv or k_cache.shape[3] != D:
        raise ValueError("k_cache must be [B, Hkv, capacity, D]")
    cap = int(k_cache.shape[2])
    n_spans = 0
    if image_spans is not None:
        _req(image_spans, "image_spans", torch.int32)
        if image_spans.dim() != 3 or image_spans.shape[0] != B or image_spans.shape[2] != 2:
            raise ValueError("image_spans must be [B, n, 2]")
        n_spans = int(image_spans.shape[1])
        if n_spans == 0:
            image_spans = None
    if out is None:
        out = torch.empty_like(q)
    _req(out, "out", torch.bfloat16, (B, C, Hq, D))
    lse = torch.empty(B, Hq, C, dtype=torch.float32, device=q.device) if return_lse else None
    need = prefill_chunk_workspace_size(B, C, Hq, Hkv, D, start, layer_kind, window)
    if need == 0:
        raise ValueError("invalid sizes for prefill_chunk")
    dev = q.device
    _on_device(dev, k=k, v=v, q_gamma=q_gamma, k_gamma=k_gamma, positions=positions, k_cache=k_cache,
               v_cache=v_cache, image_spans=image_spans, out=out)
    wsb, ws_bytes = _ws(ws, need, dev, stream=stream)
    with torch.cuda.device(dev):
        st = lib().g3attn_prefill_chunk(_ptr(q), _ptr(k), _ptr(v), _ptr(q_gamma), _ptr(k_gamma), _ptr(positions),
                                        _ptr(k_cache), _ptr(v_cache), cap, int(start), int(layer_kind),
                                        int(window), float(rope_base), float(interp_factor), _ptr(image_spans),
                                        n_spans, B, C, Hq, Hkv, D, _ptr(out), _ptr(lse), wsb.data_ptr(),
                                        ws_bytes, _stream_ptr(stream, dev))
    _check(st, "g3attn_prefill_chunk")
    return (out, lse) if return_lse else out


def soft_tokens(patches, gamma, grid_h: int, grid_w: int, pool: int = 4, *, out=None, stream=None):
    """Image soft tokens: pool x pool average of the patch grid, then RMS norm times gamma.

    patches bf16 [B, grid_h*grid_w, F], gamma fp32 [F]; returns bf16 [B, (grid_h/pool)*(grid_w/pool), F].
    """
    torch = _torch()
    _req(patches, "patches", torch.bfloat16)
    if patches.dim() != 3 or patches.shape[1] != grid_h * grid_w:
        raise ValueError("patches must be [B, grid_h * grid_w, F]")
    B, _, F = patches.shape
    _req(gamma, "gamma", torch.float32, (F,))
    n_out = (grid_h // pool) * (grid_w // pool)
    if out is None:
        out = torch.empty(B, n_out, F, dtype=torch.bfloat16, device=patches.device)
    _req(out, "out", torch.bfloat16, (B, n_out, F))
    dev = patches.device
    _on_device(dev, gamma=gamma, out=out)
    with torch.cuda.device(dev):
        st = lib().g3attn_soft_tokens(_ptr(patches), _ptr(gamma), B, grid_h, grid_w, F, pool, _ptr(out),
                                      _stream_ptr(stream, dev))
    _check(st, "g3attn_soft_tokens")
    return out
