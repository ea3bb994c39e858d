"""ctypes binding of libmoe (the C ABI in include/moe.h).

Argument marshalling only: every step of the decode runs in the CUDA kernels
behind the C ABI. torch supplies device memory, streams and data pointers. If
libmoe.so is missing, the first call raises. There is no fallback path.
"""
from __future__ import annotations

import ctypes
import json
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmoe.so")

MOE_OK = 0
STATUS_NAMES = {
    0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_CUDA",
    4: "MOE_ERR_OOM", 5: "MOE_ERR_NOT_LOADED", 6: "MOE_ERR_TIMEOUT", 7: "MOE_ERR_BAD_WEIGHTS",
}
MOE_FLAG_SPLIT_KERNELS = 0x1
MOE_FLAG_PRE_RMSNORM = 0x2
MOE_FLAG_SHARED_EXPERT = 0x4
MOE_FLAG_FP8_INTERMEDIATE = 0x8
MOE_FLAG_CUDA_CORES = 0x10
MOE_FLAG_TENSOR_CORES = 0x20
MOE_TC_MIN_TOKENS = 4
MOE_FLAG_TC_DOWN_MMA = 0x40
MOE_FLAG_TC_DOWN_CUDA = 0x80
MOE_TC_DOWN_MMA_MIN_TOKENS = 2
MOE_FLAG_SPLITK_DOWN = 0x100
MOE_LOAD_BORROW = 0x0
MOE_LOAD_SKIP_VALIDATE = 0x1
MOE_LOAD_COPY_REPACK = 0x2


class MoEError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)}")


class moe_config(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int32), ("inter", ctypes.c_int32), ("num_experts", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("max_tokens", ctypes.c_int32), ("flags", ctypes.c_uint32),
                ("device", ctypes.c_int32), ("shard_index", ctypes.c_int32), ("shard_count", ctypes.c_int32)]


_lib = None
_vp = ctypes.c_void_p


def lib() -> ctypes.CDLL:
    """Load libmoe.so (built in-tree by mxfp4_weight_streaming_fp8_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libmoe.so not found at {LIB_PATH}: build it with "
                               "`python -m mxfp4_weight_streaming_fp8_b200.build` (no fallback path exists)")
        L = ctypes.CDLL(LIB_PATH)
        L.moe_create.argtypes = [ctypes.POINTER(moe_config), ctypes.POINTER(_vp)]
        L.moe_create.restype = ctypes.c_int
        L.moe_load_experts.argtypes = [_vp] * 6 + [ctypes.c_uint32]
        L.moe_load_experts.restype = ctypes.c_int
        L.moe_decode.argtypes = [_vp, _vp, ctypes.c_int32, _vp, _vp, _vp, _vp, _vp, _vp, _vp]
        L.moe_decode.restype = ctypes.c_int
        L.moe_sync_status.argtypes = [_vp, _vp]
        L.moe_sync_status.restype = ctypes.c_int
        L.moe_query.argtypes = [_vp, ctypes.c_char_p, ctypes.c_size_t]
        L.moe_query.restype = ctypes.c_int
        L.moe_destroy.argtypes = [_vp]
        L.moe_destroy.restype = None
        L.moe_status_string.argtypes = [ctypes.c_int]
        L.moe_status_string.restype = ctypes.c_char_p
        L.moe_plan_query.argtypes = [ctypes.POINTER(moe_config), ctypes.c_int32, ctypes.c_size_t,
                                     ctypes.c_char_p, ctypes.c_size_t]
        L.moe_plan_query.restype = ctypes.c_int
        L.moe_round_bf16.argtypes = [_vp, _vp, ctypes.c_int64, _vp]
        L.moe_round_bf16.restype = ctypes.c_int
        L.moe_decode_static.argtypes = [ctypes.POINTER(moe_config)] + [_vp] * 6 + [ctypes.c_int32] + [_vp] * 6
        L.moe_decode_static.restype = ctypes.c_int
        L.moe_debug_set_wait.argtypes = [_vp, ctypes.c_longlong, ctypes.c_int]
        L.moe_debug_set_wait.restype = ctypes.c_int
        L.moe_debug_set_trace.argtypes = [_vp, _vp]
        L.moe_debug_set_trace.restype = ctypes.c_int
        L.moe_lm_create.argtypes = [ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                    ctypes.POINTER(_vp)]
        L.moe_lm_create.restype = ctypes.c_int
        L.moe_lm_load.argtypes = [_vp, _vp]
        L.moe_lm_load.restype = ctypes.c_int
        L.moe_lm_head.argtypes = [_vp, _vp, ctypes.c_int32, _vp, _vp]
        L.moe_lm_head.restype = ctypes.c_int
        L.moe_lm_sync_status.argtypes = [_vp, _vp]
        L.moe_lm_sync_status.restype = ctypes.c_int
        L.moe_lm_read_weights.argtypes = [_vp, _vp, _vp, _vp]
        L.moe_lm_read_weights.restype = ctypes.c_int
        L.moe_lm_query.argtypes = [_vp, ctypes.c_char_p, ctypes.c_size_t]
        L.moe_lm_query.restype = ctypes.c_int
        L.moe_lm_destroy.argtypes = [_vp]
        L.moe_lm_destroy.restype = None
        _lib = L
    return _lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def plan_query(hidden, inter, num_experts, top_k, max_tokens, flags=0, sm_count=148, smem_limit=232448,
               shard=(0, 1)):
    """(status, plan dict) of the persistent kernel for a shape (for part
    shard[0] of an intra-expert split over shard[1] GPUs); host only."""
    cfg = moe_config(hidden, inter, num_experts, top_k, max_tokens, flags, 0, shard[0], shard[1])
    buf = ctypes.create_string_buffer(4096)
    st = lib().moe_plan_query(ctypes.byref(cfg), sm_count, smem_limit, buf, len(buf))
    return st, (json.loads(buf.value.decode()) if buf.value else None)


def decode_static(hidden, inter, num_experts, top_k, router_w, w13_codes, w13_scales, w2_codes, w2_scales, x, M, y,
                  stream=None, topk_ids=None, topk_w=None, xq=None, xscale=None) -> int:
    """moe_decode_static: one step with no context and no allocation; returns
    the status code. Scratch is the library's fixed device array."""
    cfg = moe_config(hidden, inter, num_experts, top_k, max(1, int(M)), 0, 0)
    return lib().moe_decode_static(ctypes.byref(cfg), _ptr(router_w), _ptr(w13_codes), _ptr(w13_scales),
                                   _ptr(w2_codes), _ptr(w2_scales), _ptr(x), int(M), _ptr(y),
                                   _stream_handle(stream), _ptr(topk_ids), _ptr(topk_w), _ptr(xq), _ptr(xscale))


def round_bf16(y32, y=None, stream=None):
    """moe_round_bf16: bf16 y (same shape) from the fp32 sum of an
    intra-expert split's parts."""
    import torch
    if y is None:
        y = torch.empty(y32.shape, dtype=torch.bfloat16, device=y32.device)
    if y32.dtype != torch.float32 or y.dtype != torch.bfloat16 or y.numel() != y32.numel():
        raise ValueError("round_bf16 takes fp32 in and bf16 out of the same size")
    st = lib().moe_round_bf16(_ptr(y32), _ptr(y), y32.numel(), _stream_handle(stream))
    if st != MOE_OK:
        raise MoEError(st, "moe_round_bf16")
    return y


def decode_split(layer, x, group=None, y32=None, y=None, stream=None):
    """One step of an intra-expert split, on this rank's part `layer` (a
    MoELayer created with shard=(rank, world)): the part's fp32 sums
    (moe_decode), their sum over the ranks of `group` (one all-reduce through
    torch.distributed, NCCL on GPUs), and the bf16 round (moe_round_bf16).
    Every rank of the group must call it with the same x."""
    import torch
    import torch.distributed as dist
    if stream is not None:
        with torch.cuda.stream(stream):
            return decode_split(layer, x, group, y32, y)
    y32 = layer.decode(x, y32)
    dist.all_reduce(y32, op=dist.ReduceOp.SUM, group=group)
    return round_bf16(y32, y)


def status_string(s: int) -> str:
    return lib().moe_status_string(int(s)).decode()


class MoELayer:
    """One MoE layer's context: moe_create / moe_load_experts / moe_decode."""

    def __init__(self, hidden: int, inter: int, num_experts: int, top_k: int, max_tokens: int,
                 flags: int = 0, device: int = 0, shard=(0, 1)):
        """shard=(g, G): part g of an intra-expert split over G GPUs; decode
        then returns the part's fp32 sums (see decode_split)."""
        self.cfg = moe_config(hidden, inter, num_experts, top_k, max_tokens, flags, device, shard[0], shard[1])
        self.shard = (int(shard[0]), max(1, int(shard[1])))
        self.hidden, self.inter, self.num_experts, self.top_k = hidden, inter, num_experts, top_k
        self.max_tokens = max_tokens
        self.device = device
        self._ctx = _vp()
        st = lib().moe_create(ctypes.byref(self.cfg), ctypes.byref(self._ctx))
        if st != MOE_OK:
            raise MoEError(st, "moe_create")
        self._weights = None

    def load_experts(self, router_w, w13_codes, w13_scales, w2_codes, w2_scales, validate: bool = True,
                     repack: bool = False):
        """Borrow device tensors (kept referenced here so they outlive the
        context), or with repack=True let the context copy (and re-tile) them.
        A part of an intra-expert split always copies its slice."""
        repack = repack or self.shard[1] > 1
        flags = (0 if validate else MOE_LOAD_SKIP_VALIDATE) | (MOE_LOAD_COPY_REPACK if repack else 0)
        st = lib().moe_load_experts(self._ctx, _ptr(router_w), _ptr(w13_codes), _ptr(w13_scales),
                                    _ptr(w2_codes), _ptr(w2_scales), flags)
        if st != MOE_OK:
            raise MoEError(st, "moe_load_experts")
        self._weights = None if repack else (router_w, w13_codes, w13_scales, w2_codes, w2_scales)

    def decode_raw(self, x, M: int, y, stream=None, topk_ids=None, topk_w=None, xq=None, xscale=None,
                   xnorm=None) -> int:
        """moe_decode with explicit buffers (y: bf16 [M][H], fp32 for a part of a
        split; sizes are the caller's to get right); returns the status code."""
        return lib().moe_decode(self._ctx, _ptr(x), int(M), _ptr(y), _stream_handle(stream), _ptr(topk_ids),
                                _ptr(topk_w), _ptr(xq), _ptr(xscale), _ptr(xnorm))

    def decode(self, x, y=None, stream=None, routing: bool = False):
        """x: bf16 [M, H] on the device. Returns y, or with routing=True
        (y, topk_ids, topk_w, xq, xscale[, xnorm when the context normalises]).
        For a part of an intra-expert split y is fp32: the part's sums."""
        import torch
        M = x.shape[0]
        ydt = torch.float32 if self.shard[1] > 1 else torch.bfloat16
        if y is None:
            y = torch.empty(x.shape, dtype=ydt, device=x.device)
        elif y.dtype != ydt or y.numel() < M * self.hidden or not y.is_contiguous():
            raise ValueError(f"y must be a contiguous {ydt} tensor of at least {M} x {self.hidden} elements")
        extra = [None] * 4
        if routing:
            dev = x.device
            extra = [torch.empty((M, self.top_k), dtype=torch.int32, device=dev),
                     torch.empty((M, self.top_k), dtype=torch.float32, device=dev),
                     torch.empty((M, self.hidden), dtype=torch.uint8, device=dev),
                     torch.empty((M,), dtype=torch.float32, device=dev)]
            if self.cfg.flags & MOE_FLAG_PRE_RMSNORM:
                extra.append(torch.empty_like(x))
        st = self.decode_raw(x, M, y, stream, *extra)
        if st != MOE_OK:
            raise MoEError(st, "moe_decode")
        return (y, *extra) if routing else y

    def sync_status(self, stream=None) -> int:
        return lib().moe_sync_status(self._ctx, _stream_handle(stream))

    def set_wait(self, budget_cycles: int, force_stall: bool = False) -> int:
        return lib().moe_debug_set_wait(self._ctx, int(budget_cycles), int(bool(force_stall)))

    TRACE_SLOTS = 64  # timestamps per CTA the kernels may write

    def set_trace(self, trace) -> int:
        """Per-CTA phase timestamps of the persistent kernels into a device
        int64/uint64 tensor of at least grid x 64 words (None turns it off)."""
        if trace is not None:
            need = self.query()["grid"][0] * self.TRACE_SLOTS
            if trace.numel() < need or trace.element_size() != 8:
                raise ValueError(f"trace needs {need} 8-byte words")
        return lib().moe_debug_set_trace(self._ctx, _ptr(trace))

    def query(self) -> dict:
        buf = ctypes.create_string_buffer(1024)
        st = lib().moe_query(self._ctx, buf, len(buf))
        if st != MOE_OK:
            raise MoEError(st, "moe_query")
        return json.loads(buf.value.decode())

    def close(self):
        if self._ctx:
            lib().moe_destroy(self._ctx)
            self._ctx = _vp()
        self._weights = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class LMHead:
    """FP8 LM head context: moe_lm_create / moe_lm_load / moe_lm_head."""

    def __init__(self, vocab: int, hidden: int, max_tokens: int = 1, device: int = 0):
        self.vocab, self.hidden, self.max_tokens, self.device = vocab, hidden, max_tokens, device
        self._lm = _vp()
        st = lib().moe_lm_create(vocab, hidden, max_tokens, device, ctypes.byref(self._lm))
        if st != MOE_OK:
            raise MoEError(st, "moe_lm_create")

    def load(self, w_bf16):
        """Quantise the bf16 [vocab, hidden] device matrix into the context."""
        st = lib().moe_lm_load(self._lm, _ptr(w_bf16))
        if st != MOE_OK:
            raise MoEError(st, "moe_lm_load")

    def weights(self, stream=None):
        """(codes uint8 [vocab, hidden], scales float32 [vocab]) as device tensors (copies)."""
        import torch
        dev = f"cuda:{self.device}"
        codes = torch.empty((self.vocab, self.hidden), dtype=torch.uint8, device=dev)
        scales = torch.empty(self.vocab, dtype=torch.float32, device=dev)
        st = lib().moe_lm_read_weights(self._lm, _ptr(codes), _ptr(scales), _stream_handle(stream))
        if st != MOE_OK:
            raise MoEError(st, "moe_lm_read_weights")
        return codes, scales

    def head_raw(self, x, M: int, logits, stream=None) -> int:
        return lib().moe_lm_head(self._lm, _ptr(x), int(M), _ptr(logits), _stream_handle(stream))

    def __call__(self, x, logits=None, stream=None):
        """x: bf16 [M, hidden] on the device -> fp32 logits [M, vocab]."""
        import torch
        M = x.shape[0]
        if logits is None:
            logits = torch.empty((M, self.vocab), dtype=torch.float32, device=x.device)
        st = self.head_raw(x, M, logits, stream)
        if st != MOE_OK:
            raise MoEError(st, "moe_lm_head")
        return logits

    def sync_status(self, stream=None) -> int:
        return lib().moe_lm_sync_status(self._lm, _stream_handle(stream))

    def query(self) -> dict:
        buf = ctypes.create_string_buffer(1024)
        st = lib().moe_lm_query(self._lm, buf, len(buf))
        if st != MOE_OK:
            raise MoEError(st, "moe_lm_query")
        return json.loads(buf.value.decode())

    def close(self):
        if self._lm:
            lib().moe_lm_destroy(self._lm)
            self._lm = _vp()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
