"""Python binding of the C ABI in include/moe.h (argument marshalling only).

Every function has the name of the C entry point it calls.  Tensors are torch
tensors on the current CUDA device (bf16 as torch.bfloat16); outputs are
allocated with torch when not given.  Each call runs on the current torch CUDA
stream unless ``stream`` is given.  A non-OK status raises ``MoEError``.  There
is no fallback: without the built library every call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe_b200.so")
_lib = None

STATUS = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_WORKSPACE",
          4: "MOE_ERR_CUDA", 5: "MOE_ERR_DEVICE"}
DEVERR = {0: "MOE_DEVERR_NONE", 1: "MOE_DEVERR_BAD_EXPERT_INDEX", 2: "MOE_DEVERR_PIPELINE_TIMEOUT",
          3: "MOE_DEVERR_BAD_OFFSETS"}
MOE_DEVERR_NONE, MOE_DEVERR_BAD_EXPERT_INDEX, MOE_DEVERR_PIPELINE_TIMEOUT, MOE_DEVERR_BAD_OFFSETS = 0, 1, 2, 3
PHASES = ("route", "permute", "gemm13", "gemm2", "shared", "combine")


class MoEError(RuntimeError):
    def __init__(self, fn: str, status: int):
        detail = ""
        if status == 4:
            detail = ": " + lib().moe_last_cuda_error().decode()
        super().__init__(f"{fn} returned {STATUS.get(status, status)}{detail}")
        self.status = status


def lib() -> ctypes.CDLL:
    """Load libmoe_b200.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"CUDA library not built: {_LIB_PATH} is missing "
                               "(run __graft_entry__.build() or python expert_ffn_layer_moe_b200/build.py)")
        L = ctypes.CDLL(_LIB_PATH)
        vp, i64, c_int, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
        L.moe_status_string.argtypes = [c_int]
        L.moe_status_string.restype = ctypes.c_char_p
        L.moe_last_cuda_error.argtypes = []
        L.moe_last_cuda_error.restype = ctypes.c_char_p
        L.moe_workspace_bytes.argtypes = [i64, c_int, c_int, c_int, c_int, c_int]
        L.moe_workspace_bytes.restype = sz
        L.moe_route.argtypes = [vp, vp, vp, i64, c_int, c_int, c_int, vp, vp, vp, vp, sz, vp]
        L.moe_permute.argtypes = [vp, vp, i64, c_int, c_int, c_int, vp, vp, vp, vp, vp, vp, sz, vp]
        L.moe_permute_noalloc.argtypes = [vp, vp, i64, c_int, c_int, c_int, vp, vp, vp, vp, vp, vp]
        L.moe_expert_ffn.argtypes = [vp, vp, vp, vp, vp, i64, c_int, c_int, c_int, vp, vp, sz, vp]
        L.moe_combine.argtypes = [vp, vp, vp, vp, i64, c_int, c_int, vp, vp]
        L.moe_layer_forward.argtypes = [vp, vp, vp, vp, vp, i64, c_int, c_int, c_int, c_int, vp]
        L.moe_layer_forward_ex.argtypes = ([vp] * 9 + [i64] + [c_int] * 5 + [vp, vp, vp, sz, vp, vp])
        L.moe_get_device_error.argtypes = [vp, ctypes.POINTER(ctypes.c_int32)]
        L.moe_device_sm_count.argtypes = []
        L.moe_device_sm_count.restype = c_int
        L.moe_kernel_launches.argtypes = []
        L.moe_kernel_launches.restype = ctypes.c_uint64
        L.moe_quantize_fp8.argtypes = [vp, i64, c_int, vp, vp, vp]
        L.moe_expert_ffn_fp8.argtypes = [vp] * 8 + [i64, c_int, c_int, c_int, vp, vp, sz, vp]
        L.moe_layer_forward_fp8_ex.argtypes = ([vp] * 12 + [i64] + [c_int] * 5 + [vp, vp, vp, sz, vp, vp])
        L.moe_expert_ffn_w8a8_ws_bytes.argtypes = [i64, c_int, c_int]
        L.moe_expert_ffn_w8a8_ws_bytes.restype = sz
        L.moe_expert_ffn_w8a8.argtypes = [vp] * 8 + [i64, c_int, c_int, c_int, vp, vp, vp, sz, vp]
        L.moe_workspace_bytes_w8a8.argtypes = [i64, c_int, c_int, c_int, c_int, c_int]
        L.moe_workspace_bytes_w8a8.restype = sz
        L.moe_layer_forward_w8a8_ex.argtypes = ([vp] * 12 + [i64] + [c_int] * 5 + [vp, vp, vp, sz, vp, vp])
        L.moe_scatter_rows.argtypes = [vp, vp, i64, c_int, vp, i64, vp]
        L.moe_set_gather_mode.argtypes = [c_int]
        L.moe_set_gather_mode.restype = c_int
        L.moe_set_microbatches.argtypes = [c_int]
        L.moe_set_microbatches.restype = c_int
        L.moe_set_shared_stream.argtypes = [c_int]
        L.moe_set_shared_stream.restype = c_int
        L.moe_set_decode_gemv.argtypes = [c_int]
        L.moe_set_decode_gemv.restype = c_int
        L.moe_ipc_export.argtypes = [vp, vp, ctypes.POINTER(sz)]
        L.moe_ipc_import.argtypes = [vp, sz, ctypes.POINTER(vp)]
        L.moe_ipc_close.argtypes = [vp, sz]
        L.moe_copy_async.argtypes = [vp, vp, sz, vp]
        for fn in ("moe_ipc_export", "moe_ipc_import", "moe_ipc_close", "moe_copy_async"):
            getattr(L, fn).restype = c_int
        for fn in ("moe_route", "moe_permute", "moe_permute_noalloc", "moe_expert_ffn", "moe_combine", "moe_layer_forward",
                   "moe_layer_forward_ex", "moe_get_device_error", "moe_quantize_fp8", "moe_expert_ffn_fp8",
                   "moe_layer_forward_fp8_ex", "moe_expert_ffn_w8a8", "moe_layer_forward_w8a8_ex",
                   "moe_scatter_rows"):
            getattr(L, fn).restype = c_int
        _lib = L
    return _lib


def _p(t: Optional[torch.Tensor]):
    if t is None:
        return None
    assert t.is_contiguous(), "tensors passed to the MoE library must be contiguous"
    return ctypes.c_void_p(t.data_ptr())


def _s(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(fn: str, status: int):
    if status != 0:
        raise MoEError(fn, status)


def _empty(shape, dtype, like):
    return torch.empty(shape, dtype=dtype, device=like.device)


def moe_workspace_bytes(N: int, H: int, I: int, E: int, k: int, Is: int = 0) -> int:
    return int(lib().moe_workspace_bytes(N, H, I, E, k, Is))


def moe_device_sm_count() -> int:
    return int(lib().moe_device_sm_count())


MOE_IPC_HANDLE_BYTES = 64


def moe_ipc_export(t: torch.Tensor):
    """-> (handle bytes, byte offset) naming the device memory of tensor t for
    another process (moe_ipc_import)."""
    h = ctypes.create_string_buffer(MOE_IPC_HANDLE_BYTES)
    off = ctypes.c_size_t(0)
    _check("moe_ipc_export", lib().moe_ipc_export(_p(t), h, ctypes.byref(off)))
    return h.raw, int(off.value)


def moe_ipc_import(handle: bytes, offset: int) -> int:
    """Another process's exported buffer -> a device pointer (int) in this process."""
    ptr = ctypes.c_void_p(0)
    _check("moe_ipc_import", lib().moe_ipc_import(ctypes.create_string_buffer(handle, MOE_IPC_HANDLE_BYTES),
                                                  offset, ctypes.byref(ptr)))
    return int(ptr.value)


def moe_ipc_close(ptr: int, offset: int) -> None:
    _check("moe_ipc_close", lib().moe_ipc_close(ctypes.c_void_p(ptr), offset))


def moe_copy_async(dst_ptr: int, src_ptr: int, nbytes: int, stream=None) -> None:
    """nbytes from device pointer src_ptr to device pointer dst_ptr (ints), async."""
    _check("moe_copy_async", lib().moe_copy_async(ctypes.c_void_p(dst_ptr), ctypes.c_void_p(src_ptr), nbytes,
                                                  _s(stream)))


MOE_GATHER_AUTO, MOE_GATHER_OFF, MOE_GATHER_ON = 0, 1, 2


def moe_set_gather_mode(mode: int) -> int:
    """How the bf16 layer feeds W1/W3 its token rows: MOE_GATHER_AUTO (by shape),
    MOE_GATHER_OFF (permuted copy x_perm), MOE_GATHER_ON (gathered from x).  Returns
    the previous mode."""
    prev = int(lib().moe_set_gather_mode(int(mode)))
    if prev < 0:
        raise ValueError(f"gather mode {mode} is not one of MOE_GATHER_AUTO/OFF/ON")
    return prev


def moe_set_microbatches(m: int) -> int:
    """Run large layer calls as m (1 or 2) micro-batches on two streams; returns the
    previous value."""
    prev = int(lib().moe_set_microbatches(int(m)))
    if prev < 0:
        raise ValueError(f"micro-batches must be 1 or 2, not {m}")
    return prev


def moe_set_shared_stream(on: bool) -> bool:
    """Run the shared experts on a second stream beside the dispatch; returns the
    previous setting."""
    return bool(lib().moe_set_shared_stream(1 if on else 0))


MOE_DECODE_AUTO, MOE_DECODE_OFF, MOE_DECODE_ON = 0, 1, 2
MOE_DECODE_MAX_ROWS = 512
MOE_DECODE_MAX_TOKENS = 64


def moe_set_decode_gemv(mode: int) -> int:
    """How bf16 layer calls run the expert FFN of decode batches: MOE_DECODE_AUTO (the
    CUDA-core GEMV kernels for 2*N*k <= E, H <= 2048, I <= 1024), MOE_DECODE_OFF
    (always the grouped GEMMs), MOE_DECODE_ON (the GEMV kernels whenever N*k <=
    MOE_DECODE_MAX_ROWS).  Returns the previous mode."""
    prev = int(lib().moe_set_decode_gemv(int(mode)))
    if prev < 0:
        raise ValueError(f"decode mode {mode} is not one of MOE_DECODE_AUTO/OFF/ON")
    return prev


def moe_kernel_launches() -> int:
    """Kernels the library has launched in this process (host-side count)."""
    return int(lib().moe_kernel_launches())


def moe_route(x, W_gate, k, bias=None, logits=None, topk_idx=None, topk_w=None, ws=None, stream=None,
              use_workspace=True):
    """-> (topk_idx [N,k] int32, topk_w [N,k] fp32, logits [N,E] fp32 or None).
    With use_workspace (default) a scratch buffer is passed, which lets large
    batches take the tensor-core path; use_workspace=False runs the one-kernel
    CUDA-core path."""
    N, H = x.shape
    E = W_gate.shape[1]
    topk_idx = _empty((N, k), torch.int32, x) if topk_idx is None else topk_idx
    topk_w = _empty((N, k), torch.float32, x) if topk_w is None else topk_w
    if ws is None and use_workspace:
        ws = _empty((max(16, moe_workspace_bytes(N, H, 64, E, k, 0)),), torch.uint8, x)
    _check("moe_route", lib().moe_route(_p(x), _p(W_gate), _p(bias), N, H, E, k, _p(logits),
                                        _p(topk_idx), _p(topk_w), _p(ws), 0 if ws is None else ws.numel(),
                                        _s(stream)))
    return topk_idx, topk_w, logits


def moe_permute(x, topk_idx, E, ws=None, stream=None, out=None):
    """-> dict(counts, offsets, row_to_token, token_to_row, x_perm)."""
    N, H = x.shape
    k = topk_idx.shape[1]
    R = N * k
    o = out or {}
    # only the outputs the caller did not supply are allocated
    counts = o["counts"] if "counts" in o else _empty((E,), torch.int32, x)
    offsets = o["offsets"] if "offsets" in o else _empty((E + 1,), torch.int32, x)
    r2t = o["row_to_token"] if "row_to_token" in o else _empty((R,), torch.int32, x)
    t2r = o["token_to_row"] if "token_to_row" in o else _empty((N, k), torch.int32, x)
    x_perm = o["x_perm"] if "x_perm" in o else _empty((R, H), torch.bfloat16, x)
    if ws is None:
        ws = _empty((max(1, moe_workspace_bytes(N, H, 64, E, k, 0)),), torch.uint8, x)
    _check("moe_permute", lib().moe_permute(_p(x), _p(topk_idx), N, H, E, k, _p(counts), _p(offsets),
                                            _p(r2t), _p(t2r), _p(x_perm), _p(ws), ws.numel(), _s(stream)))
    return dict(counts=counts, offsets=offsets, row_to_token=r2t, token_to_row=t2r, x_perm=x_perm)


def moe_permute_noalloc(x, topk_idx, E, out, stream=None):
    """moe_permute without a workspace, for callers that cannot allocate device
    memory: the caller passes every output in `out` (keys counts, offsets,
    row_to_token, token_to_row, x_perm); the library's fixed scratch array is used."""
    N, H = x.shape
    k = topk_idx.shape[1]
    _check("moe_permute_noalloc", lib().moe_permute_noalloc(
        _p(x), _p(topk_idx), N, H, E, k, _p(out["counts"]), _p(out["offsets"]), _p(out["row_to_token"]),
        _p(out["token_to_row"]), _p(out["x_perm"]), _s(stream)))
    return out


def moe_expert_ffn(x_perm, offsets, W1, W3, W2, ws=None, y_perm=None, stream=None):
    """-> y_perm [R,H] fp32 (rows past offsets[E] are left as allocated)."""
    R, H = x_perm.shape
    E, I, _ = W1.shape
    y_perm = _empty((R, H), torch.float32, x_perm) if y_perm is None else y_perm
    if ws is None:
        ws = _empty((max(16, R * I * 2),), torch.uint8, x_perm)
    _check("moe_expert_ffn", lib().moe_expert_ffn(_p(x_perm), _p(offsets), _p(W1), _p(W3), _p(W2), R, H,
                                                  I, E, _p(y_perm), _p(ws), ws.numel(), _s(stream)))
    return y_perm


def moe_combine(y_perm, token_to_row, topk_w, shared_out=None, out=None, stream=None):
    """y_perm [R,H] fp32, shared_out [N,H] fp32 or None -> out [N,H] bf16."""
    N, k = token_to_row.shape
    H = y_perm.shape[1]
    out = _empty((N, H), torch.bfloat16, y_perm) if out is None else out
    _check("moe_combine", lib().moe_combine(_p(y_perm), _p(token_to_row), _p(topk_w), _p(shared_out), N,
                                            H, k, _p(out), _s(stream)))
    return out


def moe_layer_forward(x, W_gate, W1, W3, W2, k, out=None):
    """Short form: legacy default stream, library workspace; x and out may be
    CPU tensors (host buffers, copied by the call) or CUDA tensors."""
    N, H = x.shape
    E, I, _ = W1.shape
    if out is None:
        out = torch.empty((N, H), dtype=torch.bfloat16, device=x.device,
                          pin_memory=(x.device.type == "cpu"))
    _check("moe_layer_forward", lib().moe_layer_forward(_p(x), _p(W_gate), _p(W1), _p(W3), _p(W2), N, H,
                                                        I, E, k, _p(out)))
    return out


def moe_layer_forward_ex(x, W_gate, W1, W3, W2, k, bias=None, Ws1=None, Ws3=None, Ws2=None, ws=None,
                         out=None, logits=None, stream=None, phase_events: Optional[Sequence] = None):
    """Explicit form: everything on `stream` (default: current), caller's workspace."""
    N, H = x.shape
    E, I, _ = W1.shape
    Is = 0 if Ws1 is None else Ws1.shape[0]
    out = _empty((N, H), torch.bfloat16, x) if out is None else out
    if ws is None:
        ws = _empty((max(16, moe_workspace_bytes(N, H, I, E, k, Is)),), torch.uint8, x)
    ev = None
    if phase_events is not None:
        assert len(phase_events) == len(PHASES) + 1
        ev = (ctypes.c_void_p * len(phase_events))(*[e.cuda_event for e in phase_events])
    _check("moe_layer_forward_ex", lib().moe_layer_forward_ex(
        _p(x), _p(W_gate), _p(bias), _p(W1), _p(W3), _p(W2), _p(Ws1), _p(Ws3), _p(Ws2), N, H, I, E, k, Is,
        _p(out), _p(logits), _p(ws), ws.numel(), _s(stream), ev))
    return out


def moe_quantize_fp8(W, stream=None):
    """bf16 weights [..., K] -> (e4m3 bytes [..., K] uint8, fp32 scale per row [...])."""
    K = W.shape[-1]
    rows = W.numel() // K
    q = torch.empty(W.shape, dtype=torch.uint8, device=W.device)
    sc = torch.empty(W.shape[:-1], dtype=torch.float32, device=W.device)
    _check("moe_quantize_fp8", lib().moe_quantize_fp8(_p(W), rows, K, _p(q), _p(sc), _s(stream)))
    return q, sc


def moe_expert_ffn_fp8(x_perm, offsets, W1q, s1, W3q, s3, W2q, s2, ws=None, y_perm=None, stream=None):
    """moe_expert_ffn with e4m3 weights and per-row scales -> y_perm [R,H] fp32."""
    R, H = x_perm.shape
    E, I, _ = W1q.shape
    y_perm = _empty((R, H), torch.float32, x_perm) if y_perm is None else y_perm
    if ws is None:
        ws = _empty((max(16, R * I * 2),), torch.uint8, x_perm)
    _check("moe_expert_ffn_fp8", lib().moe_expert_ffn_fp8(
        _p(x_perm), _p(offsets), _p(W1q), _p(s1), _p(W3q), _p(s3), _p(W2q), _p(s2), R, H, I, E, _p(y_perm),
        _p(ws), ws.numel(), _s(stream)))
    return y_perm


def moe_layer_forward_fp8_ex(x, W_gate, W1q, s1, W3q, s3, W2q, s2, k, bias=None, Ws1=None, Ws3=None, Ws2=None,
                             ws=None, out=None, logits=None, stream=None,
                             phase_events: Optional[Sequence] = None):
    """moe_layer_forward_ex with e4m3 routed-expert weights and their per-row scales."""
    N, H = x.shape
    E, I, _ = W1q.shape
    Is = 0 if Ws1 is None else Ws1.shape[0]
    out = _empty((N, H), torch.bfloat16, x) if out is None else out
    if ws is None:
        ws = _empty((max(16, moe_workspace_bytes(N, H, I, E, k, Is)),), torch.uint8, x)
    ev = None
    if phase_events is not None:
        assert len(phase_events) == len(PHASES) + 1
        ev = (ctypes.c_void_p * len(phase_events))(*[e.cuda_event for e in phase_events])
    _check("moe_layer_forward_fp8_ex", lib().moe_layer_forward_fp8_ex(
        _p(x), _p(W_gate), _p(bias), _p(W1q), _p(s1), _p(W3q), _p(s3), _p(W2q), _p(s2), _p(Ws1), _p(Ws3),
        _p(Ws2), N, H, I, E, k, Is, _p(out), _p(logits), _p(ws), ws.numel(), _s(stream), ev))
    return out


def moe_expert_ffn_w8a8_ws_bytes(R: int, H: int, I: int) -> int:
    return int(lib().moe_expert_ffn_w8a8_ws_bytes(R, H, I))


def moe_workspace_bytes_w8a8(N: int, H: int, I: int, E: int, k: int, Is: int = 0) -> int:
    return int(lib().moe_workspace_bytes_w8a8(N, H, I, E, k, Is))


def moe_expert_ffn_w8a8(x_perm, offsets, W1q, s1, W3q, s3, W2q, s2, ws=None, y_perm=None, h=None, stream=None):
    """moe_expert_ffn with e4m3 weights and e4m3 activations (quantized per row on the
    device) -> y_perm [R,H] fp32; h [R,I] bf16, when given, receives the SwiGLU output."""
    R, H = x_perm.shape
    E, I, _ = W1q.shape
    y_perm = _empty((R, H), torch.float32, x_perm) if y_perm is None else y_perm
    if ws is None:
        ws = _empty((max(16, moe_expert_ffn_w8a8_ws_bytes(R, H, I)),), torch.uint8, x_perm)
    _check("moe_expert_ffn_w8a8", lib().moe_expert_ffn_w8a8(
        _p(x_perm), _p(offsets), _p(W1q), _p(s1), _p(W3q), _p(s3), _p(W2q), _p(s2), R, H, I, E, _p(y_perm),
        _p(h), _p(ws), ws.numel(), _s(stream)))
    return y_perm


def moe_layer_forward_w8a8_ex(x, W_gate, W1q, s1, W3q, s3, W2q, s2, k, bias=None, Ws1=None, Ws3=None, Ws2=None,
                              ws=None, out=None, logits=None, stream=None,
                              phase_events: Optional[Sequence] = None):
    """moe_layer_forward_fp8_ex with the routed experts' activations quantized to e4m3 as well."""
    N, H = x.shape
    E, I, _ = W1q.shape
    Is = 0 if Ws1 is None else Ws1.shape[0]
    out = _empty((N, H), torch.bfloat16, x) if out is None else out
    if ws is None:
        ws = _empty((max(16, moe_workspace_bytes_w8a8(N, H, I, E, k, Is)),), torch.uint8, x)
    ev = None
    if phase_events is not None:
        assert len(phase_events) == len(PHASES) + 1
        ev = (ctypes.c_void_p * len(phase_events))(*[e.cuda_event for e in phase_events])
    _check("moe_layer_forward_w8a8_ex", lib().moe_layer_forward_w8a8_ex(
        _p(x), _p(W_gate), _p(bias), _p(W1q), _p(s1), _p(W3q), _p(s3), _p(W2q), _p(s2), _p(Ws1), _p(Ws3),
        _p(Ws2), N, H, I, E, k, Is, _p(out), _p(logits), _p(ws), ws.numel(), _s(stream), ev))
    return out


def moe_scatter_rows(src, dst_row, dst, stream=None):
    """dst[dst_row[i]] = src[i] for rows with 0 <= dst_row[i] < len(dst) (bf16 or fp32 rows, on the device)."""
    assert src.dtype == dst.dtype and src.dtype in (torch.bfloat16, torch.float32) and src.shape[1:] == dst.shape[1:]
    rows = src.shape[0]
    width = src.shape[1] * (2 if src.dtype == torch.float32 else 1)
    _check("moe_scatter_rows", lib().moe_scatter_rows(_p(src), _p(dst_row), rows, width, _p(dst), dst.shape[0],
                                                      _s(stream)))
    return dst


def moe_get_device_error(stream=None) -> int:
    """Synchronise the stream, then read and clear the device error word."""
    code = ctypes.c_int32(0)
    _check("moe_get_device_error", lib().moe_get_device_error(_s(stream), ctypes.byref(code)))
    return int(code.value)
