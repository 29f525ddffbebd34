"""B200 (sm_100a) tiled exact attention: a thin ctypes binding over libfa_b200.so.

Every step of the computation runs in the CUDA library's kernels; this module
only checks tensor shapes, allocates outputs and workspaces with torch, and
passes raw device pointers and the current CUDA stream to the C ABI declared
in ``include/fa.h``.  There is no CPU fallback: if the library or a CUDA
device is missing, calls raise.

Functions (names follow the C ABI):
    forward(q, k, v, causal=False, window=0, scale=None)        -> (o, lse)
    decode(q, kcache, vcache, seqlens, scale=None)               -> (o, lse)
    decode_paged(q, kpool, vpool, block_table, seqlens)          -> (o, lse)
    backward(q, k, v, o, dout, lse, causal=False, window=0,
             scale=None)                                         -> (dq, dk, dv)
    forward_offset(q, k, v, q_offset, causal=False, window=0)   -> (o, lse)
    merge(o_parts, lse_parts)                                    -> (o, lse)
    forward_host(...)  -- forward on pinned host tensors (copies in and out)
    forward_backward_host(...)  -- forward and backward on pinned host tensors
    attention(q, k, v, causal=False, window=0, scale=None)      -> o, differentiable
    device_status()    -- FA_OK or the first recorded device-side timeout

The ring (context-parallel) forward over torch.distributed ranks sits in
``context_parallel``; its compute is ``forward_offset`` and ``merge``.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfa_b200.so")

FA_OK, FA_ERR_INVALID, FA_ERR_UNSUPPORTED, FA_ERR_CUDA, FA_ERR_TIMEOUT = range(5)
FA_BF16, FA_FP32, FA_FP16 = 0, 1, 2

EXPORTED_SYMBOLS = (
    "fa_forward",
    "fa_forward_offset",
    "fa_merge",
    "fa_decode_workspace_size",
    "fa_decode",
    "fa_decode_noalloc",
    "fa_decode_paged",
    "fa_backward_workspace_size",
    "fa_backward",
    "fa_get_device_status",
    "fa_selftest_wait_timeout",
    "fa_selftest_exp2_poly",
    "fa_status_string",
    "fa_version",
)


class FAError(RuntimeError):
    """A non-FA_OK status from the C ABI."""

    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib().fa_status_string(status).decode() if _LIB is not None else str(status)
        super().__init__(f"{where}: {msg}")


_LIB = None


def _lib() -> ctypes.CDLL:
    global _LIB
    if _LIB is not None:
        return _LIB
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m tiled_exact_attention_forward_b200.build`"
        )
    lib = ctypes.CDLL(LIB_PATH)
    P, I, F, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.fa_forward.argtypes = [P, P, P, P, P, I, I, I, I, F, I, I, I, P]
    lib.fa_forward.restype = I
    lib.fa_forward_offset.argtypes = [P, P, P, P, P, I, I, I, I, I, I, F, I, I, I, P]
    lib.fa_forward_offset.restype = I
    lib.fa_merge.argtypes = [P, P, I, P, P, I, I, I, I, I, P]
    lib.fa_merge.restype = I
    lib.fa_decode_workspace_size.argtypes = [I, I, I, I]
    lib.fa_decode_workspace_size.restype = Z
    lib.fa_decode.argtypes = [P, P, P, P, P, P, I, I, I, I, F, I, P, Z, P]
    lib.fa_decode.restype = I
    lib.fa_decode_noalloc.argtypes = [P, P, P, P, P, P, I, I, I, I, F, I, P]
    lib.fa_decode_noalloc.restype = I
    lib.fa_decode_paged.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, F, I, P, Z, P]
    lib.fa_decode_paged.restype = I
    lib.fa_backward_workspace_size.argtypes = [I, I, I, I]
    lib.fa_backward_workspace_size.restype = Z
    lib.fa_backward.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I, F, I, I, I, P, Z, P]
    lib.fa_backward.restype = I
    lib.fa_selftest_wait_timeout.argtypes = [ctypes.c_longlong, P]
    lib.fa_selftest_wait_timeout.restype = I
    lib.fa_selftest_exp2_poly.argtypes = [P, P, ctypes.c_longlong, P]
    lib.fa_selftest_exp2_poly.restype = I
    lib.fa_get_device_status.argtypes = [P]
    lib.fa_get_device_status.restype = I
    lib.fa_status_string.argtypes = [I]
    lib.fa_status_string.restype = ctypes.c_char_p
    lib.fa_version.argtypes = []
    lib.fa_version.restype = I
    _LIB = lib
    return lib


def library() -> ctypes.CDLL:
    """The loaded C library (raises ImportError if it has not been built)."""
    return _lib()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _check(status: int, where: str):
    if status != FA_OK:
        raise FAError(status, where)


def _dtype_code(dt: torch.dtype) -> int:
    if dt == torch.bfloat16:
        return FA_BF16
    if dt == torch.float16:
        return FA_FP16
    if dt == torch.float32:
        return FA_FP32
    raise TypeError(f"unsupported dtype {dt}: use torch.bfloat16, torch.float16 or torch.float32")


def _need_cuda(*ts):
    for t in ts:
        if not t.is_cuda:
            raise ValueError("tensors must be on a CUDA device (there is no CPU path)")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
        if t.device != ts[0].device:
            raise ValueError("tensors must all be on the same CUDA device")


def _scale_arg(scale) -> float:
    return 0.0 if scale is None else float(scale)


def forward(q, k, v, causal: bool = False, window: int = 0, scale=None, out=None, lse=None):
    """O = softmax(q k^T * scale + mask) v and the float32 row logsumexp.

    q, k, v: [B, H, N, d] contiguous CUDA tensors (bf16 or fp16 with d = 128, or
    fp32 with d in {64, 128}).  Returns (o, lse) with o like q and lse [B, H, N].
    """
    _need_cuda(q, k, v)
    B, H, N, d = q.shape
    if k.shape != q.shape or v.shape != q.shape or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v must share shape and dtype")
    o = torch.empty_like(q) if out is None else out
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    st = _lib().fa_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d,
                           _scale_arg(scale), int(bool(causal)), int(window),
                           _dtype_code(q.dtype), _stream(q.device))
    _check(st, "fa_forward")
    return o, lse


def forward_offset(q, k, v, q_offset: int, causal: bool = False, window: int = 0, scale=None,
                   out=None, lse=None):
    """One key shard's partial forward (context parallelism).

    q: [B, H, Nq, d]; k, v: [B, H, Nk, d] (bf16 or fp16, d = 128), contiguous CUDA
    tensors.  Query row i sits at position i + q_offset of the key sequence; the
    causal and window masks are taken at those positions.  Returns (o, lse): the
    softmax over these keys only, o like q, lse [B, H, Nq] (-inf, with o = 0, for
    a row that sees none of the keys).
    """
    _need_cuda(q, k, v)
    B, H, Nq, d = q.shape
    if k.dim() != 4 or k.shape[:2] != (B, H) or k.shape[3] != d or v.shape != k.shape:
        raise ValueError("k and v must be [B, H, Nk, d] with q's B, H and d")
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v must share dtype")
    Nk = k.shape[2]
    o = torch.empty_like(q) if out is None else out
    if lse is None:
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    st = _lib().fa_forward_offset(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, Nq, Nk,
                                  int(q_offset), d, _scale_arg(scale), int(bool(causal)), int(window),
                                  _dtype_code(q.dtype), _stream(q.device))
    _check(st, "fa_forward_offset")
    return o, lse


def merge(o_parts, lse_parts, out=None, lse=None):
    """Combine S partial results over disjoint key sets into the full attention.

    o_parts: [S, B, H, N, d] (bf16, fp16 or float32, d in {64, 128}); lse_parts:
    [S, B, H, N] float32 (-inf marks a part that saw no key for that row).
    Returns (o [B, H, N, d] in the parts' dtype, lse [B, H, N]).
    """
    _need_cuda(o_parts, lse_parts)
    S, B, H, N, d = o_parts.shape
    if lse_parts.shape != (S, B, H, N) or lse_parts.dtype != torch.float32:
        raise ValueError("lse_parts must be float32 [S, B, H, N] matching o_parts")
    o = torch.empty(o_parts.shape[1:], dtype=o_parts.dtype, device=o_parts.device) if out is None else out
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=o_parts.device)
    st = _lib().fa_merge(_ptr(o_parts), _ptr(lse_parts), S, _ptr(o), _ptr(lse), B, H, N, d,
                         _dtype_code(o_parts.dtype), _stream(o_parts.device))
    _check(st, "fa_merge")
    return o, lse


_HOST_STREAMS = {}


def _host_streams(dev):
    """Three side streams per device (copy in, compute, copy out), made once."""
    key = dev.index if dev.index is not None else torch.cuda.current_device()
    if key not in _HOST_STREAMS:
        _HOST_STREAMS[key] = tuple(torch.cuda.Stream(device=dev) for _ in range(3))
    return _HOST_STREAMS[key]


def _host_pipelined(dev, host_ins, out_specs, chunks, compute):
    """Runs `compute` over head groups with the copies pipelined around it.

    host_ins: host tensors whose first dimension is the B * H heads; out_specs:
    (trailing shape, dtype) of each output, also head-major.  For each group of
    heads [a, b): the inputs are copied in on one stream, compute(a, b, dev_ins,
    dev_outs) runs on a second, the outputs are copied back on a third, so the
    copy-in of one group overlaps the kernels of the previous group and the
    copy-out of the one before (PCIe moves both directions at once).  The
    copy-in stream first waits for the work already queued on the current
    stream; the call returns once the results are in (pinned) host memory.
    """
    BH = host_ins[0].shape[0]
    chunks = max(1, min(int(chunks), BH))
    dev_ins = [torch.empty(t.shape, dtype=t.dtype, device=dev) for t in host_ins]
    dev_outs = [torch.empty((BH, *tail), dtype=dt, device=dev) for tail, dt in out_specs]
    host_outs = [torch.empty((BH, *tail), dtype=dt, pin_memory=True) for tail, dt in out_specs]
    s_in, s_run, s_out = _host_streams(dev)
    cur = torch.cuda.current_stream(dev)
    s_in.wait_stream(cur)
    bounds = [(g * BH) // chunks for g in range(chunks + 1)]
    for g in range(chunks):
        a, b = bounds[g], bounds[g + 1]
        with torch.cuda.stream(s_in):
            for dst, src in zip(dev_ins, host_ins):
                dst[a:b].copy_(src[a:b], non_blocking=True)
        s_run.wait_stream(s_in)
        with torch.cuda.stream(s_run):
            compute(a, b, dev_ins, dev_outs)
        s_out.wait_stream(s_run)
        with torch.cuda.stream(s_out):
            for dst, src in zip(host_outs, dev_outs):
                dst[a:b].copy_(src[a:b], non_blocking=True)
    cur.wait_stream(s_out)
    s_out.synchronize()
    return host_outs, max(bounds[g + 1] - bounds[g] for g in range(chunks))


def _check_host(*ts):
    for t in ts:
        if t.is_cuda or not t.is_contiguous():
            raise ValueError("host-buffer calls take contiguous host tensors")
    if any(t.shape != ts[0].shape or t.dtype != ts[0].dtype for t in ts):
        raise ValueError("q, k, v (and dout) must share shape and dtype")


def forward_host(q, k, v, causal: bool = False, window: int = 0, scale=None, device="cuda", chunks: int = 4):
    """The forward for host tensors: copy in, run, copy out; returns pinned host (o, lse).

    q, k, v: contiguous [B, H, N, d] host tensors (pinned memory makes the copies
    asynchronous).  Every (batch, head) is independent, so the heads go through
    in `chunks` groups with copies and kernels overlapped (see _host_pipelined).
    """
    _check_host(q, k, v)
    dev = torch.device(device)
    B, H, N, d = q.shape

    def run(a, b, ins, outs):
        qd, kd, vd = (t[a:b].unsqueeze(0) for t in ins)
        forward(qd, kd, vd, causal, window, scale, out=outs[0][a:b].unsqueeze(0), lse=outs[1][a:b].unsqueeze(0))

    (o, lse), _ = _host_pipelined(dev, [t.reshape(B * H, N, d) for t in (q, k, v)],
                                  [((N, d), q.dtype), ((N,), torch.float32)], chunks, run)
    return o.view(B, H, N, d), lse.view(B, H, N)


def forward_backward_host(q, k, v, dout, causal: bool = False, window: int = 0, scale=None, device="cuda",
                          chunks: int = 8):
    """Forward and backward for host tensors; returns pinned host (o, lse, dq, dk, dv).

    The heads go through in `chunks` groups with copies and kernels overlapped
    (see _host_pipelined); the backward's workspace is sized for the largest
    group and reused, the groups' kernels running in order on one stream.
    """
    _check_host(q, k, v, dout)
    dev = torch.device(device)
    B, H, N, d = q.shape
    chunks = max(1, min(int(chunks), B * H))
    largest = -(-(B * H) // chunks)
    ws = torch.empty(max(backward_workspace_size(1, largest, N, d), 256), dtype=torch.uint8, device=dev)

    def run(a, b, ins, outs):
        qd, kd, vd, gd = (t[a:b].unsqueeze(0) for t in ins)
        od, ld, dqd, dkd, dvd = (t[a:b].unsqueeze(0) for t in outs)
        forward(qd, kd, vd, causal, window, scale, out=od, lse=ld)
        backward(qd, kd, vd, od, gd, ld, causal, window, scale, workspace=ws, dq=dqd, dk=dkd, dv=dvd)

    specs = [((N, d), q.dtype), ((N,), torch.float32)] + [((N, d), q.dtype)] * 3
    outs, _ = _host_pipelined(dev, [t.reshape(B * H, N, d) for t in (q, k, v, dout)], specs, chunks, run)
    o, lse, dq, dk, dv = outs
    return o.view(B, H, N, d), lse.view(B, H, N), dq.view(B, H, N, d), dk.view(B, H, N, d), dv.view(B, H, N, d)


def decode_workspace_size(B, H, cap, d) -> int:
    return int(_lib().fa_decode_workspace_size(B, H, cap, d))


def decode(q, kcache, vcache, seqlens, scale=None, workspace=None, out=None, lse=None):
    """Single-token decode: q [B, H, d] against kcache/vcache [B, H, cap, d].

    seqlens: int32 [B] CUDA tensor; query (b, h) attends to cache rows
    j < seqlens[b].  Returns (o [B, H, d] bf16, lse [B, H] float32).
    """
    _need_cuda(q, kcache, vcache, seqlens)
    B, H, d = q.shape
    cap = kcache.shape[2]
    if kcache.shape != (B, H, cap, d) or vcache.shape != kcache.shape:
        raise ValueError("kcache/vcache must be [B, H, cap, d] matching q")
    if kcache.dtype != q.dtype or vcache.dtype != q.dtype:
        raise ValueError("kcache/vcache must have q's dtype")
    if seqlens.dtype != torch.int32 or seqlens.shape != (B,):
        raise ValueError("seqlens must be an int32 tensor of shape [B]")
    need = decode_workspace_size(B, H, cap, d)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    o = torch.empty_like(q) if out is None else out
    if lse is None:
        lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    st = _lib().fa_decode(_ptr(q), _ptr(kcache), _ptr(vcache), _ptr(seqlens), _ptr(o), _ptr(lse),
                          B, H, cap, d, _scale_arg(scale), _dtype_code(q.dtype),
                          _ptr(workspace), workspace.numel() * workspace.element_size(),
                          _stream(q.device))
    _check(st, "fa_decode")
    return o, lse


def decode_paged(q, kpool, vpool, block_table, seqlens, scale=None, workspace=None, out=None, lse=None):
    """Single-token decode against a paged cache.

    q [B, H, d]; kpool/vpool [num_blocks, H, block_size, d] (block_size a power
    of two); block_table int32 [B, max_blocks] maps sequence b's logical block t
    (keys [t * block_size, (t + 1) * block_size)) to a pool block; seqlens int32
    [B].  Returns (o [B, H, d] bf16, lse [B, H] float32).  An out-of-range block
    id of a used block is skipped and reported by device_status().
    """
    _need_cuda(q, kpool, vpool, block_table, seqlens)
    B, H, d = q.shape
    num_blocks, _, bs, _ = kpool.shape
    if kpool.shape != (num_blocks, H, bs, d) or vpool.shape != kpool.shape:
        raise ValueError("kpool/vpool must be [num_blocks, H, block_size, d] matching q")
    if kpool.dtype != q.dtype or vpool.dtype != q.dtype:
        raise ValueError("kpool/vpool must have q's dtype")
    if block_table.dtype != torch.int32 or block_table.dim() != 2 or block_table.shape[0] != B:
        raise ValueError("block_table must be an int32 tensor of shape [B, max_blocks]")
    if seqlens.dtype != torch.int32 or seqlens.shape != (B,):
        raise ValueError("seqlens must be an int32 tensor of shape [B]")
    max_blocks = block_table.shape[1]
    need = decode_workspace_size(B, H, max_blocks * bs, d)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    o = torch.empty_like(q) if out is None else out
    if lse is None:
        lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    st = _lib().fa_decode_paged(_ptr(q), _ptr(kpool), _ptr(vpool), _ptr(block_table), _ptr(seqlens),
                                _ptr(o), _ptr(lse), B, H, num_blocks, bs, max_blocks, d, _scale_arg(scale),
                                _dtype_code(q.dtype), _ptr(workspace),
                                workspace.numel() * workspace.element_size(), _stream(q.device))
    _check(st, "fa_decode_paged")
    return o, lse


def backward_workspace_size(B, H, N, d) -> int:
    return int(_lib().fa_backward_workspace_size(B, H, N, d))


def backward(q, k, v, o, dout, lse, causal: bool = False, window: int = 0, scale=None,
             workspace=None, dq=None, dk=None, dv=None):
    """Gradients (dq, dk, dv) of the forward, recomputing P from lse."""
    _need_cuda(q, k, v, o, dout, lse)
    B, H, N, d = q.shape
    for t in (k, v, o, dout):
        if t.shape != q.shape or t.dtype != q.dtype:
            raise ValueError("q, k, v, o, dout must share shape and dtype")
    if lse.shape != (B, H, N) or lse.dtype != torch.float32:
        raise ValueError("lse must be float32 [B, H, N]")
    need = backward_workspace_size(B, H, N, d)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    st = _lib().fa_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse),
                            _ptr(dq), _ptr(dk), _ptr(dv), B, H, N, d, _scale_arg(scale),
                            int(bool(causal)), int(window), _dtype_code(q.dtype),
                            _ptr(workspace), workspace.numel() * workspace.element_size(),
                            _stream(q.device))
    _check(st, "fa_backward")
    return dq, dk, dv


class _Attention(torch.autograd.Function):
    """forward keeps (q, k, v, o, lse); backward recomputes P from lse in the library."""

    @staticmethod
    def forward(ctx, q, k, v, causal, window, scale):
        o, lse = forward(q, k, v, causal, window, scale)
        ctx.save_for_backward(q, k, v, o, lse)
        ctx.mask = (causal, window, scale)
        return o

    @staticmethod
    def backward(ctx, grad_o):
        q, k, v, o, lse = ctx.saved_tensors
        causal, window, scale = ctx.mask
        dq, dk, dv = backward(q, k, v, o, grad_o.contiguous(), lse, causal, window, scale)
        return dq, dk, dv, None, None, None


def attention(q, k, v, causal: bool = False, window: int = 0, scale=None):
    """Differentiable attention: o = softmax(q k^T * scale + mask) v with autograd.

    The forward runs the library's forward and saves the row logsumexp; the
    backward runs the library's backward, which recomputes P from it (bf16,
    d = 128 for the backward).  Gradients stay on the device.
    """
    return _Attention.apply(q, k, v, bool(causal), int(window), scale)


def selftest_wait_timeout(limit_cycles: int = 20_000_000, device=None) -> int:
    """Run the failure-path self-test kernel (a bounded wait that must expire)."""
    dev = torch.device("cuda") if device is None else torch.device(device)
    return int(_lib().fa_selftest_wait_timeout(int(limit_cycles), _stream(dev)))


def device_status(device=None) -> int:
    """Synchronise the current stream and return the library's device status."""
    dev = torch.device("cuda") if device is None else torch.device(device)
    return int(_lib().fa_get_device_status(_stream(dev)))
