"""Python binding of the exact tiled masked softmax attention library.

Thin ctypes marshalling over the C ABI declared in include/attn.h: the same
entry-point names, torch tensors turned into attn_tensor views, outputs and
workspace allocated by torch on the current device, launches on torch's
current stream. All arithmetic runs in the CUDA library; there is no CPU
path. A missing or unloadable libattn.so raises immediately.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

__all__ = [
    "AllowedSet", "AttentionFunction", "AttnError", "attention", "attn_fwd", "attn_bwd", "attn_bwd_noalloc", "attn_fwd_workspace_size",
    "attn_bwd_workspace_size", "attn_get_status", "attn_selftest_wait_timeout", "attn_set_kernel_events",
    "attn_status_string",
    "attn_version", "library_path", "load_library",
]

ATTN_OK = 0
ATTN_ERR_INVALID_ARG = 1
ATTN_ERR_UNSUPPORTED = 2
ATTN_ERR_WORKSPACE = 3
ATTN_ERR_CUDA = 4
ATTN_ERR_DEVICE = 5

ATTN_DEVERR_TOPK_INDEX = 0x1
ATTN_DEVERR_OVERFLOW = 0x2
ATTN_DEVERR_TIMEOUT = 0x4
ATTN_DEVERR_TOPK_CAUSAL = 0x8

ATTN_F32 = 0
ATTN_BF16 = 1
ATTN_F16 = 2

ATTN_MASK_CAUSAL = 0x1
ATTN_MASK_WINDOW = 0x2
ATTN_MASK_BLOCK = 0x4
ATTN_MASK_TOPK = 0x8
ATTN_MASK_LENGTHS = 0x10
ATTN_MASK_STARTS = 0x20
ATTN_MASK_TOPK_CHECK_CAUSAL = 0x40
ATTN_LSE_KV_ONLY = 0x1
ATTN_LSE_NEG_LOG2 = 0x2
ATTN_BWD_DETERMINISTIC = 0x1

_HERE = os.path.dirname(os.path.abspath(__file__))


def library_path() -> str:
    return os.path.join(_HERE, "libattn.so")


class AttnTensorC(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("ndim", ctypes.c_int32),
                ("shape", ctypes.c_int64 * 4), ("stride", ctypes.c_int64 * 4)]


class AttnMaskC(ctypes.Structure):
    _fields_ = [("flags", ctypes.c_uint32), ("window_left", ctypes.c_int64),
                ("block_mask", ctypes.c_void_p), ("block_q", ctypes.c_int32),
                ("block_k", ctypes.c_int32), ("bm_stride_b", ctypes.c_int64),
                ("bm_stride_h", ctypes.c_int64), ("bm_stride_q", ctypes.c_int64),
                ("topk_idxs", ctypes.c_void_p), ("topk_stride", ctypes.c_int64),
                ("topk_max", ctypes.c_int32), ("topk_length", ctypes.c_void_p),
                ("sink", ctypes.c_void_p), ("dropout_p", ctypes.c_float),
                ("dropout_seed", ctypes.c_uint64), ("lengths", ctypes.c_void_p),
                ("starts", ctypes.c_void_p), ("starts_stride_b", ctypes.c_int64),
                ("lse_format", ctypes.c_uint32), ("bwd_flags", ctypes.c_uint32)]


_LIB = None


def load_library():
    """Load libattn.so once; raise if it is absent (no fallback exists)."""
    global _LIB
    if _LIB is not None:
        return _LIB
    path = library_path()
    if not os.path.exists(path):
        raise RuntimeError(f"CUDA library not built: {path} is missing "
                           "(run python -m exact_tiled_attention_softmax_b200.build)")
    lib = ctypes.CDLL(path)
    T, M, vp, sz = ctypes.POINTER(AttnTensorC), ctypes.POINTER(AttnMaskC), ctypes.c_void_p, ctypes.c_size_t
    lib.attn_version.restype = ctypes.c_int
    lib.attn_status_string.restype = ctypes.c_char_p
    lib.attn_status_string.argtypes = [ctypes.c_int]
    lib.attn_fwd_workspace_size.restype = sz
    lib.attn_fwd_workspace_size.argtypes = [T, T, T, M]
    lib.attn_bwd_workspace_size.restype = sz
    lib.attn_bwd_workspace_size.argtypes = [T, T, T, M]
    lib.attn_fwd.restype = ctypes.c_int
    lib.attn_fwd.argtypes = [T, T, T, M, ctypes.c_float, T, T, vp, sz, vp]
    lib.attn_bwd.restype = ctypes.c_int
    lib.attn_bwd.argtypes = [T, T, T, T, T, T, M, ctypes.c_float, T, T, T, vp, vp, sz, vp]
    lib.attn_bwd_noalloc.restype = ctypes.c_int
    lib.attn_bwd_noalloc.argtypes = [T, T, T, T, T, T, M, ctypes.c_float, T, T, T, vp, vp]
    lib.attn_get_status.restype = ctypes.c_int
    lib.attn_get_status.argtypes = [vp, vp, ctypes.POINTER(ctypes.c_uint32)]
    lib.attn_selftest_wait_timeout.restype = ctypes.c_int
    lib.attn_selftest_wait_timeout.argtypes = [vp, sz, vp]
    lib.attn_set_kernel_events.restype = ctypes.c_int
    lib.attn_set_kernel_events.argtypes = [vp, vp]
    _LIB = lib
    return lib


class AttnError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {attn_status_string(code)} (status {code})")
        self.code = code


def attn_status_string(code: int) -> str:
    return load_library().attn_status_string(int(code)).decode()


def attn_version() -> int:
    return int(load_library().attn_version())


_DTYPES = {torch.float32: ATTN_F32, torch.bfloat16: ATTN_BF16, torch.float16: ATTN_F16}


def _tensor(t: torch.Tensor | None):
    if t is None:
        return None
    if t.dim() > 4:
        raise ValueError("at most 4 dimensions")
    c = AttnTensorC()
    c.data = t.data_ptr() if t.numel() else 0
    c.dtype = _DTYPES.get(t.dtype, -1)
    c.ndim = t.dim()
    for i in range(t.dim()):
        c.shape[i] = t.shape[i]
        c.stride[i] = t.stride(i)
    return c


def _ref(c):
    return ctypes.byref(c) if c is not None else None


def _check_on(device: torch.device, *tensors) -> None:
    """Every tensor a kernel reads or writes must sit on `device`, a CUDA
    device: the library receives raw pointers and cannot tell a host
    pointer, or another GPU's, from its own."""
    if device.type != "cuda":
        raise ValueError(f"attention tensors must be CUDA tensors (got {device})")
    for t in tensors:
        if t is not None and t.device != device:
            raise ValueError(f"a tensor is on {t.device}, the query on {device}")


def _check_mask_tensor(t: torch.Tensor, name: str, dtypes, dims) -> None:
    if t.dtype not in dtypes:
        raise ValueError(f"{name}: dtype {t.dtype}, expected one of {[str(d) for d in dtypes]}")
    if t.dim() not in dims:
        raise ValueError(f"{name}: {t.dim()} dimensions, expected {' or '.join(map(str, dims))}")
    if t.numel() > 1 and t.stride(-1) != 1:
        raise ValueError(f"{name}: the innermost dimension must be contiguous")


@dataclass
class AllowedSet:
    """The allowed-set descriptor (attn_mask). Tensors must live on the GPU.

    block_mask: uint8 [nq_blocks, nk_blocks], or with leading [B, H] dims
    (size-1 dims broadcast). topk_idxs int32 [Tq, >= topk_max],
    topk_length int32 [Tq], sink float32 [Hq]. lengths int32 [B] (active
    cells per batch row, Tq == Tk); starts int32 [B, Tq] or [Tq] (lowest
    allowed key of each query row, e.g. its packed segment's first cell).
    lse_kv_only / lse_neg_log2 select the LSE format that attn_fwd writes
    and attn_bwd expects: the sink left out, and/or stored as -log2 Z.
    deterministic makes every gradient of attn_bwd bitwise reproducible.
    topk_check_causal turns on the debug check of the top-k lists against
    each token's causal position (ATTN_DEVERR_TOPK_CAUSAL in the status).
    """
    causal: bool = False
    window_left: int = 0
    block_mask: torch.Tensor | None = None
    block_q: int = 128
    block_k: int = 128
    topk_idxs: torch.Tensor | None = None
    topk_length: torch.Tensor | None = None
    topk_max: int | None = None
    sink: torch.Tensor | None = None
    dropout_p: float = 0.0
    dropout_seed: int = 0
    lengths: torch.Tensor | None = None
    starts: torch.Tensor | None = None
    lse_kv_only: bool = False
    lse_neg_log2: bool = False
    deterministic: bool = False
    topk_check_causal: bool = False

    def tensors(self) -> list:
        """The device tensors the descriptor points at."""
        return [t for t in (self.block_mask, self.topk_idxs, self.topk_length, self.sink, self.lengths,
                            self.starts) if t is not None]

    def to_c(self) -> AttnMaskC:
        """The C descriptor. Checks each tensor's dtype and rank first, since
        the library sees only its pointer and strides."""
        for t, name, dtypes, dims in (
                (self.block_mask, "block_mask", (torch.uint8, torch.bool), (2, 4)),
                (self.topk_idxs, "topk_idxs", (torch.int32,), (2,)),
                (self.topk_length, "topk_length", (torch.int32,), (1,)),
                (self.sink, "sink", (torch.float32,), (1,)),
                (self.lengths, "lengths", (torch.int32,), (1,)),
                (self.starts, "starts", (torch.int32,), (1, 2))):
            if t is not None:
                _check_mask_tensor(t, name, dtypes, dims)
        m = AttnMaskC()
        flags = 0
        if self.causal:
            flags |= ATTN_MASK_CAUSAL
        if self.window_left:
            flags |= ATTN_MASK_WINDOW
            m.window_left = int(self.window_left)
        if self.block_mask is not None:
            bm = self.block_mask
            flags |= ATTN_MASK_BLOCK
            m.block_mask = bm.data_ptr()
            m.block_q, m.block_k = int(self.block_q), int(self.block_k)
            if bm.dim() == 2:
                m.bm_stride_b = m.bm_stride_h = 0
                m.bm_stride_q = bm.stride(0)
            else:
                m.bm_stride_b = bm.stride(0) if bm.shape[0] > 1 else 0
                m.bm_stride_h = bm.stride(1) if bm.shape[1] > 1 else 0
                m.bm_stride_q = bm.stride(2)
        if self.topk_idxs is not None:
            flags |= ATTN_MASK_TOPK
            m.topk_idxs = self.topk_idxs.data_ptr()
            m.topk_stride = self.topk_idxs.stride(0)
            m.topk_max = int(self.topk_max if self.topk_max is not None else self.topk_idxs.shape[1])
            m.topk_length = self.topk_length.data_ptr() if self.topk_length is not None else 0
            if self.topk_check_causal:
                flags |= ATTN_MASK_TOPK_CHECK_CAUSAL
        if self.lengths is not None:
            flags |= ATTN_MASK_LENGTHS
            m.lengths = self.lengths.data_ptr()
        if self.starts is not None:
            st = self.starts
            if st.stride(-1) != 1:
                raise ValueError("starts rows must be contiguous")
            flags |= ATTN_MASK_STARTS
            m.starts = st.data_ptr()
            m.starts_stride_b = st.stride(0) if st.dim() == 2 and st.shape[0] > 1 else 0
        if self.sink is not None:
            m.sink = self.sink.data_ptr()
        m.lse_format = (ATTN_LSE_KV_ONLY if self.lse_kv_only else 0) | \
            (ATTN_LSE_NEG_LOG2 if self.lse_neg_log2 else 0)
        m.bwd_flags = ATTN_BWD_DETERMINISTIC if self.deterministic else 0
        m.dropout_p = float(self.dropout_p)
        m.dropout_seed = int(self.dropout_seed) & 0xFFFFFFFFFFFFFFFF
        m.flags = flags
        return m


def _stream_handle(stream) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _workspace(nbytes: int, device) -> torch.Tensor:
    # 256-byte aligned: the caching allocator hands out 512-byte aligned blocks.
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def _is_topk(allowed: AllowedSet | None) -> bool:
    return allowed is not None and allowed.topk_idxs is not None


def attn_fwd_workspace_size(q, k, v, allowed: AllowedSet | None = None) -> int:
    cq, ck, cv = _tensor(q), _tensor(k), _tensor(v)
    m = allowed.to_c() if allowed else None
    return int(load_library().attn_fwd_workspace_size(_ref(cq), _ref(ck), _ref(cv), _ref(m)))


def attn_bwd_workspace_size(q, k, v, allowed: AllowedSet | None = None) -> int:
    cq, ck, cv = _tensor(q), _tensor(k), _tensor(v)
    m = allowed.to_c() if allowed else None
    return int(load_library().attn_bwd_workspace_size(_ref(cq), _ref(ck), _ref(cv), _ref(m)))


def attn_fwd(q, k, v, allowed: AllowedSet | None = None, scale: float | None = None, *,
             out=None, lse=None, workspace=None, stream=None):
    """Forward pass. Dense: q [B,Hq,Tq,d], k [B,Hkv,Tk,d], v [B,Hkv,Tk,dv];
    with Tq != Tk query row i sits at key position i + Tk - Tq.
    Top-k: q [Tq,H,Dqk], k = KV [Tkv,Dqk], v = KV[:, :Dv].
    Returns (o, lse); lse is fp32, natural log, sink-inclusive."""
    lib = load_library()
    if scale is None:
        scale = q.shape[-1] ** -0.5
    if out is None:
        out = torch.empty(*q.shape[:-1], v.shape[-1], dtype=q.dtype, device=q.device)
    if lse is None:
        lse = torch.empty(q.shape[:-1], dtype=torch.float32, device=q.device)
    m = allowed.to_c() if allowed else None
    cq, ck, cv, co, cl = (_tensor(x) for x in (q, k, v, out, lse))
    need = lib.attn_fwd_workspace_size(_ref(cq), _ref(ck), _ref(cv), _ref(m))
    if workspace is None:
        workspace = _workspace(need, q.device)
    _check_on(q.device, k, v, out, lse, workspace, *(allowed.tensors() if allowed else ()))
    rc = lib.attn_fwd(_ref(cq), _ref(ck), _ref(cv), _ref(m), ctypes.c_float(scale), _ref(co), _ref(cl),
                      workspace.data_ptr(), workspace.numel() * workspace.element_size(), _stream_handle(stream))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_fwd")
    return out, lse


def attn_bwd(q, k, v, o, do, lse, allowed: AllowedSet | None = None, scale: float | None = None, *,
             dq=None, dk=None, dv=None, dsink=None, workspace=None, stream=None):
    """Reverse pass. Returns (dq, dk, dv, dsink). Top-k: dk is dKV [Tkv,Dqk]
    and dv is None. dsink is None unless the allowed set carries a sink."""
    lib = load_library()
    if scale is None:
        scale = q.shape[-1] ** -0.5
    topk = _is_topk(allowed)
    if dq is None:
        dq = torch.empty_like(q)
    if dk is None:
        dk = torch.empty_like(k)
    if dv is None and not topk:
        dv = torch.empty_like(v)
    if dsink is None and allowed is not None and allowed.sink is not None:
        dsink = torch.empty_like(allowed.sink, dtype=torch.float32)
    m = allowed.to_c() if allowed else None
    cq, ck, cv, co, cdo, cl = (_tensor(x) for x in (q, k, v, o, do, lse))
    cdq, cdk, cdv = _tensor(dq), _tensor(dk), _tensor(dv)
    need = lib.attn_bwd_workspace_size(_ref(cq), _ref(ck), _ref(cv), _ref(m))
    if workspace is None:
        workspace = _workspace(need, q.device)
    _check_on(q.device, k, v, o, do, lse, dq, dk, dv, dsink, workspace,
              *(allowed.tensors() if allowed else ()))
    rc = lib.attn_bwd(_ref(cq), _ref(ck), _ref(cv), _ref(co), _ref(cdo), _ref(cl), _ref(m),
                      ctypes.c_float(scale), _ref(cdq), _ref(cdk), _ref(cdv),
                      dsink.data_ptr() if dsink is not None else None,
                      workspace.data_ptr(), workspace.numel() * workspace.element_size(), _stream_handle(stream))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_bwd")
    return dq, dk, (None if topk else dv), dsink


def attn_bwd_noalloc(q, k, v, o, do, lse, allowed: AllowedSet | None = None, scale: float | None = None, *,
                     dq, dk, dv=None, dsink=None, stream=None):
    """Reverse pass whose scratch is the library's fixed 64 MiB device array
    (for callers that cannot allocate device memory). The caller passes every
    output buffer; nothing is allocated here or in the library. Returns
    (dq, dk, dv, dsink)."""
    lib = load_library()
    if scale is None:
        scale = q.shape[-1] ** -0.5
    m = allowed.to_c() if allowed else None
    cq, ck, cv, co, cdo, cl = (_tensor(x) for x in (q, k, v, o, do, lse))
    cdq, cdk, cdv = _tensor(dq), _tensor(dk), _tensor(dv)
    _check_on(q.device, k, v, o, do, lse, dq, dk, dv, dsink, *(allowed.tensors() if allowed else ()))
    rc = lib.attn_bwd_noalloc(_ref(cq), _ref(ck), _ref(cv), _ref(co), _ref(cdo), _ref(cl), _ref(m),
                              ctypes.c_float(scale), _ref(cdq), _ref(cdk), _ref(cdv),
                              dsink.data_ptr() if dsink is not None else None, _stream_handle(stream))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_bwd_noalloc")
    return dq, dk, dv, dsink


def attn_get_status(workspace: torch.Tensor | None, stream=None) -> int:
    """Synchronise and return (then clear) the device status bits of a
    workspace, or with workspace=None those of attn_bwd_noalloc's fixed
    scratch array on the current device."""
    bits = ctypes.c_uint32(0)
    ptr = workspace.data_ptr() if workspace is not None else None
    rc = load_library().attn_get_status(ptr, _stream_handle(stream), ctypes.byref(bits))
    if rc not in (ATTN_OK, ATTN_ERR_DEVICE):
        raise AttnError(rc, "attn_get_status")
    return int(bits.value)


def attn_selftest_wait_timeout(workspace: torch.Tensor, stream=None) -> None:
    """Enqueue the failure-detection self-test: a wait that nothing completes
    runs out after its limit (2 s) and sets ATTN_DEVERR_TIMEOUT in the status
    word of `workspace` (a device tensor of at least 256 bytes); read it with
    attn_get_status."""
    rc = load_library().attn_selftest_wait_timeout(workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                                   _stream_handle(stream))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_selftest_wait_timeout")


def attn_set_kernel_events(begin: "torch.cuda.Event | None", end: "torch.cuda.Event | None") -> None:
    """Have the next attn_fwd / attn_bwd call on this thread record `begin`
    and `end` around its main kernel (timing events created with
    enable_timing=True). Each event is recorded once here first so that its
    CUDA handle exists; None, None cancels."""
    if begin is None or end is None:
        load_library().attn_set_kernel_events(None, None)
        return
    for ev in (begin, end):
        if not ev.cuda_event:
            ev.record()
    load_library().attn_set_kernel_events(ctypes.c_void_p(begin.cuda_event), ctypes.c_void_p(end.cuda_event))


class AttentionFunction(torch.autograd.Function):
    """attn_fwd / attn_bwd as one autograd node. Saves Q, K, V, O and the LSE
    (never P); the reverse pass recomputes the scores tile by tile.

    Inputs: q, k, v, sink (float32 [Hq] or None, so that its gradient is
    routed), the allowed set and the scale. Outputs: O and the LSE; the LSE is
    not differentiable through this node. Top-k (shared KV): pass k = KV and
    v = KV[:, :Dv]; the whole dKV comes back as k's gradient and v's is None,
    so a KV leaf that both were sliced from receives the tied gradient once.
    """

    @staticmethod
    def forward(ctx, q, k, v, sink, allowed, scale):
        import dataclasses
        al = dataclasses.replace(allowed, sink=sink.detach() if sink is not None else None)
        o, lse = attn_fwd(q, k, v, al, scale)
        ctx.save_for_backward(q, k, v, o, lse)
        ctx.allowed, ctx.scale, ctx.has_sink = al, scale, sink is not None
        ctx.mark_non_differentiable(lse)
        return o, lse

    @staticmethod
    def backward(ctx, d_o, d_lse):
        q, k, v, o, lse = ctx.saved_tensors
        dq, dk, dv, dsink = attn_bwd(q, k, v, o, d_o.contiguous(), lse, ctx.allowed, ctx.scale)
        return dq, dk, dv, (dsink if ctx.has_sink else None), None, None


def attention(q, k, v, allowed: AllowedSet | None = None, scale: float | None = None, sink=None):
    """Differentiable exact masked attention: returns (O, LSE). The allowed
    set's own sink field is ignored here; pass the sink tensor as `sink`."""
    if scale is None:
        scale = q.shape[-1] ** -0.5
    return AttentionFunction.apply(q, k, v, sink, allowed if allowed is not None else AllowedSet(), scale)
