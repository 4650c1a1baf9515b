"""bca_step_attend_noalloc through the C ABI.

Some callers cannot allocate device memory (their memory belongs to another
allocator, or their budget is fixed at start-up), so they cannot hand
bca_step_attend a workspace.  The no-allocation entry point uses a scratch array
inside the library instead.  Two calls in a row must give the same output as the
existing entry point with its own workspace, within the parity tolerance.  This file
is collected last on purpose, and works alone in a fresh process too."""
import ctypes
import math

import numpy as np
import pytest
import torch

import block_causal_attention_dit_b200 as bca
from block_causal_attention_dit_b200.workloads import randn_bf16
from _parity import assert_parity

pytestmark = pytest.mark.gpu


def test_noalloc_matches_workspace_entry_point_twice(cuda_device):
    L = bca.lib()
    L.bca_step_attend_noalloc.restype = ctypes.c_int
    L.bca_step_attend_noalloc.argtypes = [ctypes.c_void_p] * 4 + [
        ctypes.c_void_p, ctypes.POINTER(bca.SlotStruct), ctypes.c_int32, ctypes.c_int32,
        ctypes.c_int32, ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p]
    # 512 units on 148 SMs: the last round is split, so the scratch is really used.
    H, T, P = 32, 4096, 512
    scale = 1.0 / math.sqrt(128)
    q, k, v = (randn_bf16((T, H, 128), 7000 + t, cuda_device) for t in range(3))
    pk, pv = (randn_bf16((P, H, 128), 7010 + t, cuda_device) for t in range(2))
    slot = bca.KVSlot(P, H, "bf16")
    bca.kv_store(pk, pv, P, slot, epoch=1)
    ws = bca.step_workspace(cuda_device)
    ref = torch.empty_like(q)
    bca.step_attend(q, k, v, ref, [0, T], [slot], scale, workspace=ws)
    torch.cuda.synchronize()

    cu = (ctypes.c_int32 * 2)(0, T)
    slots = (bca.SlotStruct * 1)(slot.struct)
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    outs = [torch.full_like(q, float("nan")) for _ in range(2)]
    torch.cuda.synchronize()
    free = []
    for out in outs:
        free.append(torch.cuda.mem_get_info()[0])
        rc = L.bca_step_attend_noalloc(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                                       ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(out.data_ptr()),
                                       cu, slots, 1, H, 128, scale,
                                       ctypes.c_void_p(status.data_ptr()), stream)
        assert rc == 0, bca.status_string(rc)
        torch.cuda.synchronize()
        free.append(torch.cuda.mem_get_info()[0])
        assert int(status.item()) == 0
    # The second (warm) call took no device memory.
    assert free[3] == free[2]
    want = ref.cpu().to(torch.float64).numpy()
    for out in outs:
        assert_parity(out, want, what="noalloc vs workspace")
