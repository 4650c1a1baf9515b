"""block_causal_attention_dit_b200 -- Python binding of libbca.so.

Block-causal attention with cross-step prefix K/V reuse on B200 (sm_100a).  The
three calls of the method mirror include/bca.h one to one:

  prefill(q, k, v, o, block_offsets, scale, slot=None, epoch=0)
      step-1 block-causal attention over [S, H, 128]; optionally stores the prefix
      (every block but the last) into a KVSlot.
  kv_store(k, v, n_prefix, slot, epoch)
      prefix K/V into a KVSlot, bf16 or OFP8 E4M3 with per-head scales.
  kv_store_batch([(k, v, n_prefix, slot), ...], epoch)
      the same for the requests of a batch, in one launch.
  step_attend(q_t, k_t, v_t, o_t, cu_target, slots, scale)
      cached-step attention of packed target rows over [cache ; own K/V] for a
      ragged batch of requests at the same phase.
  step_attend_q8(q_t, k_t, v_t, o_t, cu_target, slots, scale, q8_scratch)
      the same over e4m3 ("fp8") slots with e4m3 Q against the e4m3 cached keys.
  step_attend_dq(q_t, k_t, v_t, o_t, cu_target, slots, scale, dq_scratch)
      step_attend over e4m3 slots with the cache expanded to bf16 once per call.
  qk_norm_rope(q, k, gamma_q, gamma_k, cos_t, sin_t, eps)
      Q/K RMS norm + rotary embedding of the rows entering attention (in place).
  qkv_project(x, w, q, k, v, gamma_q, gamma_k, cos_t, sin_t, eps)
      the projection of rows into Q, K, V with that norm + rotary in its epilogue.
  StepGraph(q_layers, k_layers, v_layers, o_layers, cu_target, slots_per_layer, scale)
      the cached-step calls of every layer of one layout recorded as one CUDA graph;
      .launch() replays them (bit-identical to the eager calls).

This module only marshals arguments (device pointers, sizes, the current CUDA
stream) into the C ABI: every step of the path runs in the library's kernels.
PyTorch is used for device memory and streams.  If the library is missing the
calls raise; there is no other implementation behind them.
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "BcaError", "KVSlot", "KV_BF16", "KV_FP8_V", "KV_FP8_KV", "MAX_BLOCKS", "MAX_BATCH",
    "lib", "prefill", "kv_store", "kv_store_batch", "step_attend", "step_workspace", "step_workspace_bytes",
    "step_attend_q8", "step_q8_scratch", "step_q8_scratch_bytes", "q8_views",
    "step_attend_dq", "step_dq_scratch", "step_dq_scratch_bytes",
    "StepGraph", "qk_norm_rope", "qkv_project", "ulysses_pack", "ulysses_unpack",
    "slot_bytes", "set_wait_timeout_ns",
    "selftest_wait_timeout", "selftest_e4m3_division", "status_string",
    "version", "LIB_PATH",
]

# BCA_LIBRARY may name another build of the same library (e.g. the self-checking
# libbca_checked.so); there is no other implementation behind these calls.
LIB_PATH = os.environ.get("BCA_LIBRARY") or os.path.join(
    os.path.dirname(os.path.abspath(__file__)), "libbca.so")

KV_BF16, KV_FP8_V, KV_FP8_KV = 0, 1, 2
_DTYPE_NAMES = {"bf16": KV_BF16, "fp8_v": KV_FP8_V, "fp8": KV_FP8_KV}
MAX_BLOCKS = 64
MAX_BATCH = 64

STATUS_NAMES = {
    0: "BCA_OK", 1: "BCA_ERR_INVALID_ARG", 2: "BCA_ERR_UNSUPPORTED", 3: "BCA_ERR_CAPACITY",
    4: "BCA_ERR_STATE", 5: "BCA_ERR_CUDA", 6: "BCA_ERR_DEVICE_TIMEOUT", 7: "BCA_ERR_NONFINITE",
}


class BcaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = int(status)
        super().__init__(f"{where}: {STATUS_NAMES.get(self.status, self.status)}")


class StepGraphDesc(ctypes.Structure):
    """Mirror of bca_step_graph_desc."""
    _fields_ = [
        ("n_layers", ctypes.c_int32),
        ("q_t", ctypes.POINTER(ctypes.c_void_p)), ("k_t", ctypes.POINTER(ctypes.c_void_p)),
        ("v_t", ctypes.POINTER(ctypes.c_void_p)), ("o_t", ctypes.POINTER(ctypes.c_void_p)),
        ("slots", ctypes.c_void_p), ("cu_target", ctypes.POINTER(ctypes.c_int32)),
        ("n_req", ctypes.c_int32), ("heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("scale", ctypes.c_float), ("workspace", ctypes.c_void_p),
        ("workspace_bytes", ctypes.c_size_t), ("dev_status", ctypes.c_void_p),
        ("q8_scratch", ctypes.c_void_p), ("q8_scratch_bytes", ctypes.c_size_t),
        ("dq_scratch", ctypes.c_void_p), ("dq_scratch_bytes", ctypes.c_size_t),
    ]


class SlotStruct(ctypes.Structure):
    """Mirror of bca_kv_slot."""
    _fields_ = [
        ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("k_scale", ctypes.c_void_p), ("v_scale", ctypes.c_void_p),
        ("cap_tokens", ctypes.c_int32), ("n_tokens", ctypes.c_int32),
        ("num_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("dtype", ctypes.c_int32), ("epoch", ctypes.c_uint32),
    ]


class StoreItemStruct(ctypes.Structure):
    """Mirror of bca_kv_store_item."""
    _fields_ = [
        ("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("n_prefix", ctypes.c_int32),
        ("row_stride_elems", ctypes.c_int32), ("slot", ctypes.POINTER(SlotStruct)),
    ]


_lib = None


def lib():
    """Load libbca.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing: build it with "
            "`python -m block_causal_attention_dit_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, i32, u32, u64, f32 = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_uint32,
                             ctypes.c_uint64, ctypes.c_float)
    SP = ctypes.POINTER(SlotStruct)
    L.bca_kv_slot_bytes.restype = ctypes.c_size_t
    L.bca_kv_slot_bytes.argtypes = [i32, i32, i32, ctypes.c_int]
    L.bca_kv_slot_init.restype = ctypes.c_int
    L.bca_kv_slot_init.argtypes = [SP, P, i32, i32, i32, ctypes.c_int]
    L.bca_kv_store.restype = ctypes.c_int
    L.bca_kv_store.argtypes = [P, P, i32, i32, SP, u32, P, P]
    L.bca_kv_store_batch.restype = ctypes.c_int
    L.bca_kv_store_batch.argtypes = [ctypes.POINTER(StoreItemStruct), i32, u32, P, P]
    L.bca_prefill.restype = ctypes.c_int
    L.bca_prefill.argtypes = [P, P, P, P, i32, P, i32, i32, i32, f32, SP, u32, P, P]
    L.bca_prefill_ws.restype = ctypes.c_int
    L.bca_prefill_ws.argtypes = [P, P, P, P, i32, P, i32, i32, i32, f32, SP, u32, P,
                                 ctypes.c_size_t, P, P]
    L.bca_step_attend.restype = ctypes.c_int
    L.bca_step_attend.argtypes = [P, P, P, P, P, SP, i32, i32, i32, f32, P, ctypes.c_size_t,
                                  P, P]
    L.bca_step_workspace_bytes.restype = ctypes.c_size_t
    L.bca_step_workspace_bytes.argtypes = []
    L.bca_step_attend_q8.restype = ctypes.c_int
    L.bca_step_attend_q8.argtypes = [P, P, P, P, P, SP, i32, i32, i32, f32, P, ctypes.c_size_t,
                                     P, ctypes.c_size_t, P, P]
    L.bca_step_attend_dq.restype = ctypes.c_int
    L.bca_step_attend_dq.argtypes = [P, P, P, P, P, SP, i32, i32, i32, f32, P, ctypes.c_size_t,
                                     P, ctypes.c_size_t, P, P]
    L.bca_step_dq_scratch_bytes.restype = ctypes.c_size_t
    L.bca_step_dq_scratch_bytes.argtypes = [SP, i32]
    L.bca_step_q8_scratch_bytes.restype = ctypes.c_size_t
    L.bca_step_q8_scratch_bytes.argtypes = [ctypes.c_int64, i32, i32]
    L.bca_status_string.restype = ctypes.c_char_p
    L.bca_status_string.argtypes = [ctypes.c_int]
    L.bca_set_wait_timeout_ns.restype = None
    L.bca_set_wait_timeout_ns.argtypes = [u64]
    L.bca_selftest_wait_timeout.restype = ctypes.c_int
    L.bca_selftest_wait_timeout.argtypes = [P, u64, P]
    L.bca_selftest_e4m3_division.restype = ctypes.c_int
    L.bca_selftest_e4m3_division.argtypes = [P, P]
    L.bca_debug_set_trace.restype = ctypes.c_int
    L.bca_debug_set_trace.argtypes = [P, i32]
    L.bca_qk_norm_rope.restype = ctypes.c_int
    L.bca_qk_norm_rope.argtypes = [P, P, ctypes.c_int64, i32, i32, P, P, P, P, f32, P]
    L.bca_qkv_project.restype = ctypes.c_int
    L.bca_qkv_project.argtypes = [P, P, P, P, P, i32, i32, i32, i32, P, P, P, P, f32, P, P]
    for name in ("bca_ulysses_pack", "bca_ulysses_unpack"):
        getattr(L, name).restype = ctypes.c_int
        getattr(L, name).argtypes = [P, P, ctypes.c_int64, i32, i32, i32, P]
    L.bca_step_graph_create.restype = ctypes.c_int
    L.bca_step_graph_create.argtypes = [ctypes.POINTER(StepGraphDesc), ctypes.POINTER(P)]
    L.bca_step_graph_launch.restype = ctypes.c_int
    L.bca_step_graph_launch.argtypes = [P, P]
    L.bca_step_graph_kernel_nodes.restype = i32
    L.bca_step_graph_kernel_nodes.argtypes = [P]
    L.bca_step_graph_destroy.restype = None
    L.bca_step_graph_destroy.argtypes = [P]
    L.bca_version.restype = ctypes.c_char_p
    L.bca_version.argtypes = []
    _lib = L
    return L


def _check(status: int, where: str):
    if status != 0:
        raise BcaError(status, where)


# Checks of what the C ABI cannot see (it receives bare pointers): every tensor is a
# CUDA tensor of the expected dtype, dense where the library assumes density, and
# large enough for the rows the call will read or write.  A failed check raises
# BcaError(BCA_ERR_INVALID_ARG) before anything is enqueued.
def _need(cond, call: str, what: str):
    if not cond:
        raise BcaError(1, f"{call} ({what})")


def _cuda(t, call, name, dtype=None, device=None):
    import torch
    _need(isinstance(t, torch.Tensor) and t.is_cuda, call, f"{name} must be a CUDA tensor")
    if dtype is not None:
        _need(t.dtype == dtype, call, f"{name} must be {dtype}")
    if device is not None:
        _need(t.device == device, call, f"{name} must be on {device}")


def _rows_tensor(t, call, name, like=None):
    """[rows, H, d] bf16, contiguous (the library's THD layout); `like`: same shape
    and device as that tensor."""
    import torch
    _cuda(t, call, name, torch.bfloat16, None if like is None else like.device)
    _need(t.dim() == 3 and t.is_contiguous(), call, f"{name} must be a contiguous [rows, H, d]")
    if like is not None:
        _need(t.shape == like.shape, call, f"{name} must have shape {tuple(like.shape)}")


def _aux(t, call, name, device, dtype=None, min_numel=1):
    if t is None:
        return
    _cuda(t, call, name, dtype, device)
    _need(t.is_contiguous() and t.numel() >= min_numel, call,
          f"{name} must be contiguous with at least {min_numel} elements")


def _slot_device(slot, call, device):
    _need(slot.buffer.device == device, call, f"slot buffers must be on {device}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream, device=None):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def _i32_array(values):
    vals = [int(x) for x in values]
    return (ctypes.c_int32 * len(vals))(*vals)


def status_string(status: int) -> str:
    return lib().bca_status_string(int(status)).decode()


def version() -> str:
    return lib().bca_version().decode()


def slot_bytes(cap_tokens: int, heads: int, head_dim: int = 128, dtype="bf16") -> int:
    dt = _DTYPE_NAMES.get(dtype, dtype)
    return int(lib().bca_kv_slot_bytes(cap_tokens, heads, head_dim, dt))


def set_wait_timeout_ns(ns: int):
    lib().bca_set_wait_timeout_ns(int(ns))


class KVSlot:
    """One (request, layer) prefix K/V cache slot carved from one device buffer.

    `buffer` is a torch uint8 CUDA tensor of slot_bytes(...) bytes (allocated here
    when not given); `struct` is the bca_kv_slot the library reads and updates."""

    def __init__(self, cap_tokens: int, heads: int, dtype="bf16", head_dim: int = 128,
                 device="cuda", buffer=None):
        import torch
        self.dtype = _DTYPE_NAMES.get(dtype, dtype)
        n = slot_bytes(cap_tokens, heads, head_dim, self.dtype)
        if n == 0:
            raise BcaError(1, "KVSlot")
        if buffer is None:
            buffer = torch.empty(n, dtype=torch.uint8, device=device)
        assert buffer.numel() >= n and buffer.dtype == torch.uint8
        self.buffer = buffer
        self.struct = SlotStruct()
        _check(lib().bca_kv_slot_init(ctypes.byref(self.struct), _ptr(buffer), cap_tokens,
                                      heads, head_dim, self.dtype), "bca_kv_slot_init")

    # Views of the slot's device memory (for tests and inspection).
    def _view(self, addr, nbytes, torch_dtype, shape):
        import torch
        off = addr - self.buffer.data_ptr()
        return self.buffer[off:off + nbytes].view(torch_dtype).view(*shape)

    def k_view(self):
        import torch
        s = self.struct
        fp8 = self.dtype == KV_FP8_KV
        es = 1 if fp8 else 2
        return self._view(s.k, s.num_heads * s.cap_tokens * s.head_dim * es,
                          torch.uint8 if fp8 else torch.bfloat16,
                          (s.num_heads, s.cap_tokens, s.head_dim))

    def v_view(self):
        import torch
        s = self.struct
        fp8 = self.dtype in (KV_FP8_V, KV_FP8_KV)
        es = 1 if fp8 else 2
        return self._view(s.v, s.num_heads * s.cap_tokens * s.head_dim * es,
                          torch.uint8 if fp8 else torch.bfloat16,
                          (s.num_heads, s.cap_tokens, s.head_dim))

    def k_scale_view(self):
        import torch
        return self._view(self.struct.k_scale, 4 * self.struct.num_heads, torch.float32,
                          (self.struct.num_heads,))

    def v_scale_view(self):
        import torch
        return self._view(self.struct.v_scale, 4 * self.struct.num_heads, torch.float32,
                          (self.struct.num_heads,))

    @property
    def n_tokens(self) -> int:
        return int(self.struct.n_tokens)

    @property
    def epoch(self) -> int:
        return int(self.struct.epoch)


def _store_args(call, k, v, n_prefix, slot, row_stride):
    """Checks of one store's tensors; returns the row stride in elements."""
    import torch
    for name, t in (("k", k), ("v", v)):
        _cuda(t, call, name, torch.bfloat16, k.device)
        _need(t.dim() in (2, 3) and t.stride(-1) == 1 and
              (t.dim() == 2 or t.stride(1) == t.shape[2]), call, f"{name} rows must be dense")
        width = t.shape[1] * (t.shape[2] if t.dim() == 3 else 1)
        _need(width == slot.struct.num_heads * slot.struct.head_dim, call,
              f"{name} rows must hold the slot's heads x head_dim values")
        _need(t.shape[0] >= int(n_prefix), call, f"{name} has fewer than n_prefix rows")
    if row_stride is None:
        row_stride = k.stride(0) if k.shape[0] > 1 else width
    _need(k.shape[0] <= 1 or (k.stride(0) == row_stride and v.stride(0) == row_stride), call,
          "k and v rows must be row_stride elements apart")
    _slot_device(slot, call, k.device)
    return int(row_stride)


def kv_store(k, v, n_prefix: int, slot: KVSlot, epoch: int, row_stride: int | None = None,
             dev_status=None, stream=None):
    """Prefix rows [0, n_prefix) of k and v into the slot.  k and v are bf16 CUDA
    tensors [rows, H, d] or [rows, H*d] whose rows are dense and `row_stride`
    elements apart (default: their stride(0)); both use the same row stride."""
    import torch
    call = "bca_kv_store"
    row_stride = _store_args(call, k, v, n_prefix, slot, row_stride)
    _aux(dev_status, call, "dev_status", k.device, torch.int32)
    _check(lib().bca_kv_store(_ptr(k), _ptr(v), int(n_prefix), int(row_stride),
                              ctypes.byref(slot.struct), int(epoch), _ptr(dev_status),
                              _stream(stream, k.device)), "bca_kv_store")


def kv_store_batch(items, epoch: int, dev_status=None, stream=None):
    """kv_store for several requests in one launch.  items: (k, v, n_prefix, slot) or
    (k, v, n_prefix, slot, row_stride) tuples, one per request, distinct slots."""
    import torch
    call = "bca_kv_store_batch"
    _need(len(items) >= 1, call, "at least one item")
    arr = (StoreItemStruct * len(items))()
    keep = []
    for i, it in enumerate(items):
        k, v, n_prefix, slot = it[:4]
        rs = _store_args(call, k, v, n_prefix, slot, it[4] if len(it) > 4 else None)
        _need(k.device == items[0][0].device, call, "all items on one device")
        arr[i] = StoreItemStruct(k.data_ptr(), v.data_ptr(), int(n_prefix), rs,
                                 ctypes.pointer(slot.struct))
        keep.append(slot)
    dev = items[0][0].device
    _aux(dev_status, call, "dev_status", dev, torch.int32)
    _check(lib().bca_kv_store_batch(arr, len(items), int(epoch), _ptr(dev_status),
                                    _stream(stream, dev)), call)


def prefill(q, k, v, o, block_offsets, scale: float, slot: KVSlot | None = None,
            epoch: int = 0, dev_status=None, stream=None, workspace=None):
    """Block-causal attention of [S, H, 128]; with `workspace` (step_workspace())
    through bca_prefill_ws, whose schedule splits the heavy Q-tile pairs' last round."""
    import torch
    call = "bca_prefill" if workspace is None else "bca_prefill_ws"
    _rows_tensor(q, call, "q")
    for name, t in (("k", k), ("v", v), ("o", o)):
        _rows_tensor(t, call, name, like=q)
    if slot is not None:
        _slot_device(slot, call, q.device)
    _aux(dev_status, call, "dev_status", q.device, torch.int32)
    _aux(workspace, call, "workspace", q.device)
    S, H, d = q.shape
    off = _i32_array(block_offsets)
    sl = None if slot is None else ctypes.byref(slot.struct)
    if workspace is None:
        rc = lib().bca_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(o), S, off, len(off) - 1, H, d,
                               float(scale), sl, int(epoch), _ptr(dev_status),
                               _stream(stream, q.device))
    else:
        rc = lib().bca_prefill_ws(_ptr(q), _ptr(k), _ptr(v), _ptr(o), S, off, len(off) - 1, H,
                                  d, float(scale), sl, int(epoch), _ptr(workspace),
                                  workspace.numel() * workspace.element_size(),
                                  _ptr(dev_status), _stream(stream, q.device))
    _check(rc, call)


def step_workspace_bytes() -> int:
    return int(lib().bca_step_workspace_bytes())


def step_workspace(device="cuda"):
    """A workspace for step_attend (uint8 CUDA tensor of step_workspace_bytes())."""
    import torch
    return torch.empty(max(step_workspace_bytes(), 256), dtype=torch.uint8, device=device)


def _check_step_args(call, q_t, k_t, v_t, o_t, cu_target, slots):
    _rows_tensor(q_t, call, "q_t")
    for name, t in (("k_t", k_t), ("v_t", v_t), ("o_t", o_t)):
        _rows_tensor(t, call, name, like=q_t)
    cu = [int(x) for x in cu_target]
    _need(len(cu) == len(slots) + 1, call, "cu_target needs one entry per slot plus one")
    _need(cu[-1] <= q_t.shape[0], call, "cu_target[-1] exceeds the rows of q_t")
    for sl in slots:
        _slot_device(sl, call, q_t.device)
    return cu


def step_attend(q_t, k_t, v_t, o_t, cu_target, slots, scale: float, workspace=None,
                dev_status=None, stream=None):
    import torch
    call = "bca_step_attend"
    cu = _check_step_args(call, q_t, k_t, v_t, o_t, cu_target, slots)
    _aux(workspace, call, "workspace", q_t.device)
    _aux(dev_status, call, "dev_status", q_t.device, torch.int32)
    _, H, d = q_t.shape
    cu = _i32_array(cu)
    arr = (SlotStruct * len(slots))(*[s.struct for s in slots])
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().bca_step_attend(_ptr(q_t), _ptr(k_t), _ptr(v_t), _ptr(o_t), cu, arr,
                                 len(slots), H, d, float(scale), _ptr(workspace), ws_bytes,
                                 _ptr(dev_status), _stream(stream, q_t.device)),
           "bca_step_attend")


def step_dq_scratch_bytes(slots) -> int:
    """Bytes of step_attend_dq's scratch for these (filled) slots."""
    arr = (SlotStruct * len(slots))(*[s.struct for s in slots])
    return int(lib().bca_step_dq_scratch_bytes(arr, len(slots)))


def step_dq_scratch(slots, device="cuda"):
    import torch
    return torch.empty(max(step_dq_scratch_bytes(slots), 256), dtype=torch.uint8, device=device)


def step_attend_dq(q_t, k_t, v_t, o_t, cu_target, slots, scale: float, dq_scratch=None,
                   workspace=None, dev_status=None, stream=None):
    """step_attend over e4m3 ("fp8_v" / "fp8") slots with each cache tensor expanded
    once to bf16 in dq_scratch before the attention (bit-identical results)."""
    import torch
    call = "bca_step_attend_dq"
    cu = _check_step_args(call, q_t, k_t, v_t, o_t, cu_target, slots)
    _, H, d = q_t.shape
    if dq_scratch is None:
        dq_scratch = step_dq_scratch(slots, q_t.device)
    _aux(dq_scratch, call, "dq_scratch", q_t.device)
    _aux(workspace, call, "workspace", q_t.device)
    _aux(dev_status, call, "dev_status", q_t.device, torch.int32)
    arr = (SlotStruct * len(slots))(*[s.struct for s in slots])
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().bca_step_attend_dq(_ptr(q_t), _ptr(k_t), _ptr(v_t), _ptr(o_t), _i32_array(cu),
                                    arr, len(slots), H, d, float(scale), _ptr(workspace),
                                    ws_bytes, _ptr(dq_scratch),
                                    dq_scratch.numel() * dq_scratch.element_size(),
                                    _ptr(dev_status), _stream(stream, q_t.device)), call)
    return dq_scratch


def step_q8_scratch_bytes(rows: int, n_req: int, heads: int) -> int:
    return int(lib().bca_step_q8_scratch_bytes(int(rows), int(n_req), int(heads)))


def step_q8_scratch(rows: int, n_req: int, heads: int, device="cuda"):
    """Scratch for step_attend_q8 (uint8 CUDA tensor of step_q8_scratch_bytes())."""
    import torch
    n = step_q8_scratch_bytes(rows, n_req, heads)
    if n == 0:
        raise BcaError(1, "bca_step_q8_scratch_bytes")
    return torch.empty(n, dtype=torch.uint8, device=device)


def q8_views(q8_scratch, rows: int, n_req: int, heads: int):
    """(codes [H, rows, 128] uint8, scales [n_req, H] fp32) inside a q8 scratch."""
    import torch
    nc = (heads * rows * 128 + 255) // 256 * 256
    codes = q8_scratch[:heads * rows * 128].view(heads, rows, 128)
    scales = q8_scratch[nc:nc + 4 * n_req * heads].view(torch.float32).view(n_req, heads)
    return codes, scales


def step_attend_q8(q_t, k_t, v_t, o_t, cu_target, slots, scale: float, q8_scratch=None,
                   workspace=None, dev_status=None, stream=None):
    """step_attend over "fp8" slots with e4m3 Q for the scores of cached keys (Q of
    each request quantised per head like a cache tensor, into q8_scratch)."""
    import torch
    call = "bca_step_attend_q8"
    cu = _check_step_args(call, q_t, k_t, v_t, o_t, cu_target, slots)
    _, H, d = q_t.shape
    if q8_scratch is None:
        q8_scratch = step_q8_scratch(cu[-1], len(slots), H, q_t.device)
    _aux(q8_scratch, call, "q8_scratch", q_t.device)
    _aux(workspace, call, "workspace", q_t.device)
    _aux(dev_status, call, "dev_status", q_t.device, torch.int32)
    arr = (SlotStruct * len(slots))(*[s.struct for s in slots])
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().bca_step_attend_q8(_ptr(q_t), _ptr(k_t), _ptr(v_t), _ptr(o_t), _i32_array(cu),
                                    arr, len(slots), H, d, float(scale), _ptr(workspace),
                                    ws_bytes, _ptr(q8_scratch),
                                    q8_scratch.numel() * q8_scratch.element_size(),
                                    _ptr(dev_status), _stream(stream, q_t.device)), call)
    return q8_scratch


def qk_norm_rope(q, k, gamma_q, gamma_k, cos_t, sin_t, eps: float = 1e-6, stream=None):
    """In place on q and/or k ([rows, H, 128] bf16 CUDA; either may be None):
    RMS norm over the head dim with weights gamma_* ([128] fp32), then the rotary
    embedding of channel pairs (2i, 2i+1) by the angles whose cos/sin are
    cos_t[t, i], sin_t[t, i] ([rows, 64] fp32)."""
    import torch
    call = "bca_qk_norm_rope"
    ref = q if q is not None else k
    if ref is None:
        raise BcaError(1, call)
    _rows_tensor(ref, call, "q" if q is not None else "k")
    if q is not None and k is not None:
        _rows_tensor(k, call, "k", like=q)
    rows, H, d = ref.shape
    if rows > 0:
        for name, t, x in (("gamma_q", gamma_q, q), ("gamma_k", gamma_k, k)):
            if x is not None:
                _need(t is not None, call, f"{name} is required with its tensor")
                _aux(t, call, name, ref.device, torch.float32, d)
        for name, t in (("cos_t", cos_t), ("sin_t", sin_t)):
            _need(t is not None, call, f"{name} is required")
            _aux(t, call, name, ref.device, torch.float32, rows * (d // 2))
    _check(lib().bca_qk_norm_rope(_ptr(q), _ptr(k), rows, H, d, _ptr(gamma_q), _ptr(gamma_k),
                                  _ptr(cos_t), _ptr(sin_t), float(eps),
                                  _stream(stream, ref.device)), "bca_qk_norm_rope")


def qkv_project(x, w, q, k, v, gamma_q, gamma_k, cos_t, sin_t, eps: float = 1e-6,
                dev_status=None, stream=None):
    """q, k, v ([rows, H, 128] bf16 CUDA, written) from x [rows, D] and w [3*H*128, D]
    (bf16 CUDA): the projection x w^T with the Q/K RMS norm (gamma_q / gamma_k, [128]
    fp32) and the rotary embedding (cos_t / sin_t, [rows, 64] fp32) in its epilogue."""
    import torch
    call = "bca_qkv_project"
    _cuda(x, call, "x", torch.bfloat16)
    _need(x.dim() == 2 and x.is_contiguous(), call, "x must be a contiguous [rows, D]")
    rows, D = x.shape
    _cuda(w, call, "w", torch.bfloat16, x.device)
    _need(w.dim() == 2 and w.is_contiguous() and w.shape[1] == D, call,
          "w must be a contiguous [3*H*128, D]")
    _rows_tensor(q, call, "q")
    _need(q.device == x.device and q.shape[0] == rows, call, "q must have x's rows")
    for name, t in (("k", k), ("v", v)):
        _rows_tensor(t, call, name, like=q)
    H, d = q.shape[1], q.shape[2]
    _need(w.shape[0] == 3 * H * d, call, "w must have 3*H*head_dim rows")
    for name, t, n in (("gamma_q", gamma_q, d), ("gamma_k", gamma_k, d),
                       ("cos_t", cos_t, rows * (d // 2)), ("sin_t", sin_t, rows * (d // 2))):
        _need(t is not None, call, f"{name} is required")
        _aux(t, call, name, x.device, torch.float32, n)
    _aux(dev_status, call, "dev_status", x.device, torch.int32)
    _check(lib().bca_qkv_project(_ptr(x), _ptr(w), _ptr(q), _ptr(k), _ptr(v), rows, D, H, d,
                                 _ptr(gamma_q), _ptr(gamma_k), _ptr(cos_t), _ptr(sin_t),
                                 float(eps), _ptr(dev_status), _stream(stream, x.device)), call)


def ulysses_pack(x, send, n_ranks: int, stream=None):
    """x [rows, H, 128] -> send [n_ranks, rows, H/n_ranks, 128] (block g for rank g)."""
    import torch
    _rows_tensor(x, "bca_ulysses_pack", "x")
    _aux(send, "bca_ulysses_pack", "send", x.device, torch.bfloat16, x.numel())
    rows, H, d = x.shape
    _check(lib().bca_ulysses_pack(_ptr(x), _ptr(send), rows, H, d, int(n_ranks),
                                  _stream(stream, x.device)), "bca_ulysses_pack")


def ulysses_unpack(recv, x, n_ranks: int, stream=None):
    """recv [n_ranks, rows, H/n_ranks, 128] (block g from rank g) -> x [rows, H, 128]."""
    import torch
    _rows_tensor(x, "bca_ulysses_unpack", "x")
    _aux(recv, "bca_ulysses_unpack", "recv", x.device, torch.bfloat16, x.numel())
    rows, H, d = x.shape
    _check(lib().bca_ulysses_unpack(_ptr(recv), _ptr(x), rows, H, d, int(n_ranks),
                                    _stream(stream, x.device)), "bca_ulysses_unpack")


class StepGraph:
    """The cached-step attention of every layer of one layout as one CUDA graph
    (with q8_scratch: the e4m3-Q cached step, step_attend_q8, of e4m3 slots; with
    dq_scratch: the expand-once step, step_attend_dq).

    q_layers..o_layers: per-layer packed target tensors [sum T_r, H, 128] (bf16,
    CUDA); slots_per_layer: per-layer lists of KVSlot (one per request, in
    cu_target order).  The buffers are read in place at every launch(): write new
    contents into them between launches.  Keep them (and the slots) alive while the
    graph exists; close() or garbage collection releases it."""

    def __init__(self, q_layers, k_layers, v_layers, o_layers, cu_target, slots_per_layer,
                 scale: float, workspace=None, dev_status=None, q8_scratch=None,
                 dq_scratch=None):
        n = len(q_layers)
        assert n == len(k_layers) == len(v_layers) == len(o_layers) == len(slots_per_layer)
        n_req = len(slots_per_layer[0])
        assert all(len(sl) == n_req for sl in slots_per_layer)
        import torch
        call = "bca_step_graph_create"
        for l in range(n):
            _check_step_args(call, q_layers[l], k_layers[l], v_layers[l], o_layers[l], cu_target,
                             slots_per_layer[l])
            _need(q_layers[l].shape == q_layers[0].shape, call, "layers must share one layout")
        _aux(workspace, call, "workspace", q_layers[0].device)
        _aux(dev_status, call, "dev_status", q_layers[0].device, torch.int32)
        _aux(q8_scratch, call, "q8_scratch", q_layers[0].device)
        _aux(dq_scratch, call, "dq_scratch", q_layers[0].device)
        _, H, d = q_layers[0].shape
        self._keep = (list(q_layers), list(k_layers), list(v_layers), list(o_layers),
                      [list(sl) for sl in slots_per_layer], workspace, dev_status, q8_scratch,
                      dq_scratch)
        ptrs = lambda ts: (ctypes.c_void_p * n)(*[t.data_ptr() for t in ts])
        self._q, self._k, self._v, self._o = (ptrs(q_layers), ptrs(k_layers), ptrs(v_layers),
                                              ptrs(o_layers))
        self._slots = (SlotStruct * (n * n_req))(*[s.struct for sl in slots_per_layer for s in sl])
        self._cu = _i32_array(cu_target)
        desc = StepGraphDesc(
            n, ctypes.cast(self._q, ctypes.POINTER(ctypes.c_void_p)),
            ctypes.cast(self._k, ctypes.POINTER(ctypes.c_void_p)),
            ctypes.cast(self._v, ctypes.POINTER(ctypes.c_void_p)),
            ctypes.cast(self._o, ctypes.POINTER(ctypes.c_void_p)),
            ctypes.cast(self._slots, ctypes.c_void_p), self._cu, n_req, H, d, float(scale),
            None if workspace is None else workspace.data_ptr(),
            0 if workspace is None else workspace.numel() * workspace.element_size(),
            None if dev_status is None else dev_status.data_ptr(),
            None if q8_scratch is None else q8_scratch.data_ptr(),
            0 if q8_scratch is None else q8_scratch.numel() * q8_scratch.element_size(),
            None if dq_scratch is None else dq_scratch.data_ptr(),
            0 if dq_scratch is None else dq_scratch.numel() * dq_scratch.element_size())
        self.device = q_layers[0].device
        self._g = ctypes.c_void_p()
        import torch
        with torch.cuda.device(self.device):
            _check(lib().bca_step_graph_create(ctypes.byref(desc), ctypes.byref(self._g)),
                   "bca_step_graph_create")

    @property
    def kernel_nodes(self) -> int:
        return int(lib().bca_step_graph_kernel_nodes(self._g))

    def launch(self, stream=None):
        _check(lib().bca_step_graph_launch(self._g, _stream(stream, self.device)),
               "bca_step_graph_launch")

    def close(self):
        if getattr(self, "_g", None):
            lib().bca_step_graph_destroy(self._g)
            self._g = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def selftest_wait_timeout(dev_status, timeout_ns: int, stream=None):
    _check(lib().bca_selftest_wait_timeout(_ptr(dev_status), int(timeout_ns),
                                           _stream(stream, dev_status.device)),
           "bca_selftest_wait_timeout")


def selftest_e4m3_division(device="cuda", stream=None):
    """Pairs (bf16 x, bf16 amax) whose e4m3 code from the encoder's division differs
    from the code of the correctly rounded x / (amax / 448) (0 expected)."""
    import torch
    n = torch.zeros(1, dtype=torch.int64, device=device)
    _check(lib().bca_selftest_e4m3_division(_ptr(n), _stream(stream, n.device)),
           "bca_selftest_e4m3_division")
    return int(n.item())

