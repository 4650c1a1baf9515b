"""The C ABI without a GPU: the library loads, exports every function that
include/bca.h declares, and rejects invalid arguments on the host before any CUDA
call (so these checks never touch a device)."""
import ctypes
import os
import re

import pytest

import block_causal_attention_dit_b200 as bca

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bca.h")


@pytest.fixture(scope="module")
def L():
    from block_causal_attention_dit_b200 import build
    build.build()
    return bca.lib()


def declared_functions():
    with open(HEADER) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b(bca_[a-z0-9_]+)\s*\(", text)
    return sorted(set(names))


def test_header_declares_the_three_calls():
    names = declared_functions()
    for n in ("bca_prefill", "bca_kv_store", "bca_step_attend"):
        assert n in names


def test_every_declared_symbol_is_exported(L):
    for name in declared_functions():
        assert hasattr(L, name), name


def test_status_strings(L):
    for code, name in bca.STATUS_NAMES.items():
        assert bca.status_string(code) == name
    assert "sm_100a" in bca.version()


def test_slot_bytes_and_layout(L):
    H, cap = 4, 100
    nb = bca.slot_bytes(cap, H, 128, "bf16")
    assert nb >= 2 * cap * H * 128 * 2
    assert bca.slot_bytes(cap, H, 128, "fp8") < nb
    assert bca.slot_bytes(-1, H, 128, "bf16") == 0
    assert bca.slot_bytes(cap, 0, 128, "bf16") == 0
    s = bca.SlotStruct()
    base = 1 << 20  # host-side carving only: no memory is touched
    assert L.bca_kv_slot_init(ctypes.byref(s), ctypes.c_void_p(base), cap, H, 128, bca.KV_FP8_KV) == 0
    assert s.k == base and s.v > s.k and s.k_scale > s.v and s.v_scale > s.k_scale
    assert all(x % 256 == 0 for x in (s.k, s.v, s.k_scale, s.v_scale))
    assert s.v - s.k >= cap * H * 128 and s.epoch == 0 and s.n_tokens == 0
    assert L.bca_kv_slot_init(ctypes.byref(s), ctypes.c_void_p(base + 16), cap, H, 128, 0) == 1


def _slot(L, cap=64, H=2, dt=0, epoch=1, n=10):
    s = bca.SlotStruct()
    assert L.bca_kv_slot_init(ctypes.byref(s), ctypes.c_void_p(1 << 20), cap, H, 128, dt) == 0
    s.epoch, s.n_tokens = epoch, n
    return s


FAKE = ctypes.c_void_p(1 << 24)  # never dereferenced: every case fails validation first


def test_prefill_argument_errors(L):
    off = (ctypes.c_int32 * 3)(0, 64, 128)
    args = lambda **kw: dict(dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, S=128, off=off, nb=2, H=2,
                                  d=128, scale=0.1, slot=None, epoch=0), **kw)
    call = lambda a: L.bca_prefill(a["q"], a["k"], a["v"], a["o"], a["S"], a["off"], a["nb"],
                                   a["H"], a["d"], a["scale"], a["slot"], a["epoch"], None, None)
    assert call(args(q=None)) == 1
    assert call(args(d=64)) == 2
    assert call(args(H=0)) == 1
    assert call(args(S=100)) == 1  # offsets do not end at S
    assert call(args(nb=0)) == 1
    assert call(args(scale=0.0)) == 1
    assert call(args(scale=float("nan"))) == 1
    assert call(args(q=ctypes.c_void_p((1 << 24) + 8))) == 1  # misaligned
    bad = (ctypes.c_int32 * 3)(0, 0, 128)
    assert call(args(off=bad)) == 1  # empty block
    s = _slot(L, cap=32, H=2)
    assert call(args(slot=ctypes.pointer(s), epoch=1)) == 3  # prefix 64 > cap 32
    s = _slot(L, cap=128, H=2)
    assert call(args(slot=ctypes.pointer(s), epoch=0)) == 1  # epoch 0
    s = _slot(L, cap=128, H=3)
    assert call(args(slot=ctypes.pointer(s), epoch=1)) == 1  # head mismatch


def test_kv_store_argument_errors(L):
    s = _slot(L, cap=16, H=2)
    st = lambda **kw: L.bca_kv_store(kw.get("k", FAKE), kw.get("v", FAKE), kw.get("n", 8),
                                     kw.get("stride", 256), ctypes.byref(kw.get("slot", s)),
                                     kw.get("epoch", 1), None, None)
    assert st(n=17) == 3
    assert st(n=-1) == 1
    assert st(epoch=0) == 1
    assert st(stride=128) == 1  # < heads * 128
    assert st(stride=260) == 1  # not a multiple of 8
    assert st(k=None) == 1
    assert L.bca_kv_store(FAKE, FAKE, 4, 256, None, 1, None, None) == 1
    s2 = _slot(L, cap=16, H=2, dt=2)
    s2.k_scale = None
    assert st(slot=s2) == 1
    s3 = _slot(L, cap=16, H=2)
    s3.head_dim = 64
    assert st(slot=s3) == 2


def test_kv_store_batch_argument_errors(L):
    """bca_kv_store_batch checks every item as bca_kv_store does, and that the slots
    are distinct, before anything is launched; a failed call stamps no slot."""
    slots = [_slot(L, cap=16, H=2, epoch=0, n=0) for _ in range(3)]
    Item = bca.StoreItemStruct
    mk = lambda n_prefix=8, stride=256, slot=0: Item(FAKE.value, FAKE.value, n_prefix, stride,
                                                     ctypes.pointer(slots[slot]))
    call = lambda items, epoch=1: L.bca_kv_store_batch((Item * len(items))(*items), len(items),
                                                       epoch, None, None)
    assert L.bca_kv_store_batch(None, 1, 1, None, None) == 1
    assert L.bca_kv_store_batch((Item * 1)(mk()), 0, 1, None, None) == 1
    assert call([mk(slot=i % 3) for i in range(65)]) == 1  # more than BCA_MAX_BATCH
    assert call([mk(slot=0), mk(slot=1), mk(slot=0)]) == 1  # a slot twice
    assert call([mk(slot=0), mk(n_prefix=17, slot=1)]) == 3  # beyond cap
    assert call([mk(slot=0), mk(stride=128, slot=1)]) == 1
    assert call([mk(slot=0)], epoch=0) == 1
    assert all(s.epoch == 0 and s.n_tokens == 0 for s in slots)


def test_step_attend_argument_errors(L):
    cu = (ctypes.c_int32 * 3)(0, 100, 228)
    s0, s1 = _slot(L, n=10), _slot(L, n=20)
    arr = (bca.SlotStruct * 2)(s0, s1)
    call = lambda **kw: L.bca_step_attend(FAKE, FAKE, FAKE, FAKE, kw.get("cu", cu),
                                          kw.get("arr", arr), kw.get("n", 2), kw.get("H", 2),
                                          kw.get("d", 128), kw.get("scale", 0.1),
                                          kw.get("ws", None), kw.get("ws_bytes", 0), None, None)
    assert call(d=96) == 2
    assert call(n=0) == 1
    assert call(n=65) == 1
    assert call(H=4) == 1  # slots have 2 heads
    assert call(cu=(ctypes.c_int32 * 3)(0, 100, 50)) == 1
    assert call(cu=(ctypes.c_int32 * 3)(1, 100, 228)) == 1
    empty = (bca.SlotStruct * 2)(s0, _slot(L, epoch=0))
    assert call(arr=empty) == 4
    mixed = (bca.SlotStruct * 2)(s0, _slot(L, dt=2))
    assert call(arr=mixed) == 2
    over = _slot(L, cap=64, n=65)
    assert call(arr=(bca.SlotStruct * 2)(s0, over)) == 1
    assert call(ws=ctypes.c_void_p((1 << 24) + 16), ws_bytes=1 << 20) == 1  # misaligned workspace


def test_step_attend_q8_argument_errors(L):
    """bca_step_attend_q8 checks, before anything is enqueued: e4m3 K and V slots
    (an e4m3 Q meets e4m3 K codes), a non-NULL 256-byte aligned scratch, and its
    size; bca_step_q8_scratch_bytes gives that size."""
    H, rows = 2, 228
    need = L.bca_step_q8_scratch_bytes(rows, 2, H)
    codes = (H * rows * 128 + 255) // 256 * 256
    assert need == codes + 256  # codes, then the [n_req][H] fp32 scales
    assert L.bca_step_q8_scratch_bytes(-1, 2, H) == 0
    assert L.bca_step_q8_scratch_bytes(rows, 0, H) == 0
    assert L.bca_step_q8_scratch_bytes(rows, 65, H) == 0
    assert L.bca_step_q8_scratch_bytes(rows, 2, 0) == 0
    cu = (ctypes.c_int32 * 3)(0, 100, rows)
    fp8 = (bca.SlotStruct * 2)(_slot(L, dt=2), _slot(L, dt=2, n=20))
    scratch = ctypes.c_void_p(1 << 28)
    call = lambda **kw: L.bca_step_attend_q8(
        FAKE, FAKE, FAKE, FAKE, cu, kw.get("arr", fp8), 2, H, 128, 0.1, None, 0,
        kw.get("scratch", scratch), kw.get("bytes", need), None, None)
    assert call(arr=(bca.SlotStruct * 2)(_slot(L), _slot(L, n=20))) == 2  # bf16 slots
    assert call(arr=(bca.SlotStruct * 2)(_slot(L, dt=1), _slot(L, dt=1, n=20))) == 2  # fp8_v
    assert call(scratch=None) == 1
    assert call(scratch=ctypes.c_void_p((1 << 28) + 16)) == 1  # not 256-byte aligned
    assert call(bytes=need - 1) == 3


def test_selftest_wait_rejects_bad_bounds(L):
    assert L.bca_selftest_wait_timeout(None, 10_000_000, None) == 1
    assert L.bca_selftest_wait_timeout(FAKE, 10, None) == 1


def test_step_graph_argument_errors(L):
    """bca_step_graph_create rejects a malformed description before any CUDA call."""
    cu = (ctypes.c_int32 * 2)(0, 128)
    ptrs = (ctypes.c_void_p * 2)(FAKE.value, FAKE.value)
    pp = ctypes.cast(ptrs, ctypes.POINTER(ctypes.c_void_p))
    slots = (bca.SlotStruct * 2)(_slot(L), _slot(L))
    good = dict(n_layers=2, q_t=pp, k_t=pp, v_t=pp, o_t=pp,
                slots=ctypes.cast(slots, ctypes.c_void_p), cu_target=cu, n_req=1, heads=2,
                head_dim=128, scale=0.1, workspace=None, workspace_bytes=0, dev_status=None)
    out = ctypes.c_void_p()
    create = lambda **kw: L.bca_step_graph_create(ctypes.byref(bca.StepGraphDesc(**dict(good, **kw))),
                                                  ctypes.byref(out))
    assert L.bca_step_graph_create(None, ctypes.byref(out)) == 1
    assert L.bca_step_graph_create(ctypes.byref(bca.StepGraphDesc(**good)), None) == 1
    assert create(n_layers=0) == 1
    assert create(q_t=None) == 1
    assert create(o_t=None) == 1
    assert create(slots=None) == 1
    assert create(cu_target=None) == 1
    assert create(n_req=0) == 1
    assert create(n_req=65) == 1
    assert out.value is None
    assert L.bca_step_graph_launch(None, None) == 1
    assert L.bca_step_graph_kernel_nodes(None) == 0
    L.bca_step_graph_destroy(None)


def test_qk_norm_rope_argument_errors(L):
    call = lambda **kw: L.bca_qk_norm_rope(kw.get("q", FAKE), kw.get("k", FAKE), kw.get("rows", 16),
                                           kw.get("H", 2), kw.get("d", 128), kw.get("gq", FAKE),
                                           kw.get("gk", FAKE), kw.get("c", FAKE), kw.get("s", FAKE),
                                           kw.get("eps", 1e-6), None)
    assert call(d=64) == 2
    assert call(rows=-1) == 1
    assert call(H=0) == 1
    assert call(H=257) == 1
    assert call(eps=0.0) == 1
    assert call(eps=float("nan")) == 1
    assert call(q=None, k=None) == 1
    assert call(q=None, k=None, rows=0) == 0  # nothing to do
    assert call(q=ctypes.c_void_p((1 << 24) + 8)) == 1  # misaligned
    assert call(gq=None) == 1
    assert call(k=None, gk=None, c=None) == 1
    assert call(s=ctypes.c_void_p((1 << 24) + 4)) == 1


def test_ulysses_copy_argument_errors(L):
    for fn in (L.bca_ulysses_pack, L.bca_ulysses_unpack):
        call = lambda **kw: fn(kw.get("a", FAKE), kw.get("b", FAKE), kw.get("rows", 16),
                               kw.get("H", 32), kw.get("d", 128), kw.get("n", 4), None)
        assert call(d=64) == 2
        assert call(n=0) == 1
        assert call(n=3) == 1  # 32 heads over 3 ranks
        assert call(H=0) == 1
        assert call(rows=-1) == 1
        assert call(a=None) == 1
        assert call(b=ctypes.c_void_p((1 << 24) + 8)) == 1
        assert call(a=None, rows=0) == 0  # nothing to move


def test_binding_rejects_host_tensors_before_the_library_is_called():
    """The Python binding passes bare pointers to the C ABI, so it checks what the
    ABI cannot: host (CPU) tensors are refused with BCA_ERR_INVALID_ARG before
    anything is enqueued."""
    import torch
    x = torch.zeros((4, 2, 128), dtype=torch.bfloat16)
    calls = [
        lambda: bca.step_attend(x, x, x, x, [0, 4], [], 0.1),
        lambda: bca.step_attend_q8(x, x, x, x, [0, 4], [], 0.1),
        lambda: bca.prefill(x, x, x, x, [0, 4], 0.1),
        lambda: bca.qk_norm_rope(x, None, None, None, None, None),
        lambda: bca.ulysses_pack(x, torch.empty_like(x), 2),
        lambda: bca.ulysses_unpack(torch.empty_like(x), x, 2),
    ]
    for call in calls:
        with pytest.raises(bca.BcaError) as e:
            call()
        assert e.value.status == 1 and "CUDA tensor" in str(e.value)


def test_qkv_project_argument_errors(L):
    """bca_qkv_project checks shapes, sizes and pointers before any CUDA call."""
    call = lambda **kw: L.bca_qkv_project(
        kw.get("x", FAKE), kw.get("w", FAKE), FAKE, FAKE, FAKE, kw.get("rows", 64),
        kw.get("D", 128), kw.get("H", 2), kw.get("d", 128), FAKE, FAKE, kw.get("cos", FAKE),
        FAKE, kw.get("eps", 1e-6), None, None)
    assert call(d=64) == 2
    assert call(D=100) == 2
    assert call(D=0) == 2
    assert call(rows=-1) == 1
    assert call(H=0) == 1
    assert call(H=257) == 1
    assert call(eps=0.0) == 1
    assert call(eps=float("inf")) == 1
    assert call(x=None) == 1
    assert call(w=ctypes.c_void_p((1 << 24) + 8)) == 1  # misaligned
    assert call(cos=None) == 1
    assert call(rows=0, x=None) == 0  # nothing to do, nothing checked


def test_step_attend_dq_argument_errors(L):
    """bca_step_attend_dq: e4m3 slots, a non-NULL 256-byte aligned scratch of at
    least bca_step_dq_scratch_bytes (per request: bf16 [H, n_tokens, 128] for each e4m3
    tensor, 256-byte aligned), all checked before anything is enqueued."""
    H = 2
    fp8 = (bca.SlotStruct * 2)(_slot(L, dt=2, n=10), _slot(L, dt=2, n=20))
    fp8v = (bca.SlotStruct * 2)(_slot(L, dt=1, n=10), _slot(L, dt=1, n=20))
    bf = (bca.SlotStruct * 2)(_slot(L, n=10), _slot(L, n=20))
    r256 = lambda n: (n + 255) // 256 * 256
    need = L.bca_step_dq_scratch_bytes(fp8, 2)
    assert need == 2 * r256(10 * H * 256) + 2 * r256(20 * H * 256)
    assert L.bca_step_dq_scratch_bytes(fp8v, 2) == r256(10 * H * 256) + r256(20 * H * 256)
    assert L.bca_step_dq_scratch_bytes(bf, 2) == 0
    assert L.bca_step_dq_scratch_bytes(None, 2) == 0
    assert L.bca_step_dq_scratch_bytes(fp8, 0) == 0
    cu = (ctypes.c_int32 * 3)(0, 100, 228)
    scratch = ctypes.c_void_p(1 << 28)
    call = lambda **kw: L.bca_step_attend_dq(
        FAKE, FAKE, FAKE, FAKE, cu, kw.get("arr", fp8), 2, H, 128, 0.1, None, 0,
        kw.get("scratch", scratch), kw.get("bytes", need), None, None)
    assert call(arr=bf) == 2
    assert call(scratch=None) == 1
    assert call(scratch=ctypes.c_void_p((1 << 28) + 16)) == 1
    assert call(bytes=need - 1) == 3
