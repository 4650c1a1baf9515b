"""bca_step_attend_noalloc through the C ABI.

Some callers cannot allocate device memory (their memory belongs to another
allocator, or their budget is fixed at start-up), so they cannot hand
bca_step_attend a workspace.  The no-allocation entry point uses a scratch array
inside the library instead.  It runs the same kernels with the same schedule as the
workspace entry point, so its output must equal that entry point's bit for bit; it
is also held to the oracle within the bf16 tolerance.

Two layouts are used, both with a split last round (so the scratch is really read
and written), with different numbers of split units and chunks per unit; they run
one after the other and then the first again, so each call starts from the other
layout's leftover scratch contents.  That the split path ran is checked twice: the
mirror of the library's schedule predicts a split, and the output differs from the
call without any workspace (whose last round is not split) while it equals the
workspace call.

This file is collected last on purpose, and works alone in a fresh process too."""
import ctypes
import math

import pytest
import torch

import block_causal_attention_dit_b200 as bca
import oracle
from block_causal_attention_dit_b200.workloads import randn_bf16
from _parity import assert_parity, sample_rows

pytestmark = pytest.mark.gpu
SCALE = 1.0 / math.sqrt(128)
CHUNKS = 160  # the library's array, in split chunks


def _split_k(units: int, sms: int, ws_chunks: int, min_tiles: int) -> int:
    """Chunks per split unit in the library's schedule (1: no split)."""
    if ws_chunks == 0 or units <= sms or units % sms == 0:
        return 1
    rem = units % sms
    k = min(sms // rem, 8, ws_chunks // rem, min_tiles)
    return k if k >= 2 else 1


def _layout(H, targets, prefixes, seed, device):
    reqs = []
    for i, (T, P) in enumerate(zip(targets, prefixes)):
        q, k, v = (randn_bf16((T, H, 128), seed + 10 * i + t, device) for t in range(3))
        pk, pv = (randn_bf16((P, H, 128), seed + 10 * i + 5 + t, device) for t in range(2))
        slot = bca.KVSlot(P, H, "bf16", device=device)
        bca.kv_store(pk, pv, P, slot, epoch=1)
        reqs.append(dict(q=q, k=k, v=v, pk=pk, pv=pv, slot=slot, T=T, P=P))
    cu = [0]
    for T in targets:
        cu.append(cu[-1] + T)
    cat = lambda n: torch.cat([r[n] for r in reqs])
    return dict(H=H, reqs=reqs, cu=cu, q=cat("q"), k=cat("k"), v=cat("v"))


def _noalloc(L, x, out, status):
    cu = (ctypes.c_int32 * len(x["cu"]))(*x["cu"])
    slots = (bca.SlotStruct * len(x["reqs"]))(*[r["slot"].struct for r in x["reqs"]])
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = L.bca_step_attend_noalloc(ctypes.c_void_p(x["q"].data_ptr()),
                                   ctypes.c_void_p(x["k"].data_ptr()),
                                   ctypes.c_void_p(x["v"].data_ptr()),
                                   ctypes.c_void_p(out.data_ptr()), cu, slots, len(x["reqs"]),
                                   x["H"], 128, SCALE, ctypes.c_void_p(status.data_ptr()), stream)
    assert rc == 0, bca.status_string(rc)


def test_noalloc_equals_workspace_entry_point_and_oracle(cuda_device):
    L = bca.lib()
    L.bca_step_attend_noalloc.restype = ctypes.c_int
    L.bca_step_attend_noalloc.argtypes = [ctypes.c_void_p] * 4 + [
        ctypes.c_void_p, ctypes.POINTER(bca.SlotStruct), ctypes.c_int32, ctypes.c_int32,
        ctypes.c_int32, ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p]
    sms = torch.cuda.get_device_properties(cuda_device).multi_processor_count
    assert sms <= CHUNKS
    # A: 32 heads x 16 Q-tile pairs = 512 units; B: two requests, 37 heads x (3 + 2)
    # pairs = 185 units.  On 148 SMs: A splits 68 units in 2, B 37 units in 4.
    layouts = [_layout(32, [4096], [512], 7000, cuda_device),
               _layout(37, [700, 450], [700, 333], 7100, cuda_device)]
    ws = bca.step_workspace(cuda_device)
    ws_chunks = bca.step_workspace_bytes() // (256 * 130 * 4)
    ks = []
    for x in layouts:
        units = sum(x["H"] * -(-r["T"] // 256) for r in x["reqs"])
        tiles = min(-(-r["P"] // 128) + -(-r["T"] // 128) for r in x["reqs"])
        k_ws = _split_k(units, sms, ws_chunks, tiles)
        k_na = _split_k(units, sms, CHUNKS, tiles)
        assert k_ws >= 2 and k_na == k_ws, (units, k_ws, k_na)
        ks.append(k_ws)
        x["ref"] = torch.empty_like(x["q"])
        bca.step_attend(x["q"], x["k"], x["v"], x["ref"], x["cu"],
                        [r["slot"] for r in x["reqs"]], SCALE, workspace=ws)
        x["unsplit"] = torch.empty_like(x["q"])
        bca.step_attend(x["q"], x["k"], x["v"], x["unsplit"], x["cu"],
                        [r["slot"] for r in x["reqs"]], SCALE)
    assert ks[0] != ks[1]
    torch.cuda.synchronize()

    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    free = []
    for n, x in enumerate([layouts[0], layouts[0], layouts[1], layouts[0]]):
        out = torch.full_like(x["q"], float("nan"))
        torch.cuda.synchronize()
        free.append(torch.cuda.mem_get_info()[0])
        _noalloc(L, x, out, status)
        torch.cuda.synchronize()
        free.append(torch.cuda.mem_get_info()[0])
        assert int(status.item()) == 0
        assert torch.equal(out, x["ref"]), f"call {n}: differs from the workspace call"
        assert not torch.equal(out, x["unsplit"]), f"call {n}: the last round was not split"
        x.setdefault("outs", []).append(out)
    # After the first call (which may do the one-time set-up) no call took device
    # memory: free memory is the same before and after each of them.
    for n in range(1, len(free) // 2):
        assert free[2 * n + 1] == free[2 * n], f"call {n} took device memory"
    for x in layouts:
        for r, (c0, c1) in zip(x["reqs"], zip(x["cu"], x["cu"][1:])):
            rows = sample_rows(r["T"], 96, seed=r["T"], boundaries=range(256, r["T"], 256))
            want = oracle.cached_step(r["q"].cpu(), r["k"].cpu(), r["v"].cpu(),
                                      r["pk"].cpu().permute(1, 0, 2).contiguous(),
                                      r["pv"].cpu().permute(1, 0, 2).contiguous(), r["P"],
                                      SCALE, rows=rows)
            idx = torch.from_numpy(rows).to(cuda_device)
            assert_parity(x["outs"][0][c0:c1][idx], want, what=f"noalloc T={r['T']}")
