"""One kernel of the hot path on one workload, run a few times and timed: the
command that profiles (ncu) capture, and a quick timing check.

    python -m block_causal_attention_dit_b200.profile_cases <case> [workload] [reps]

cases (workloads are those of ``workloads.workload``: 0 tiny, 1 T2I 1024x1024, 2
4-ref edit, 3 native 2K, 4 step-batched serving with an e4m3 cache):
    store    bca_kv_store_batch of every request's prefix K/V (one launch)
    prefill  bca_prefill of request 0 (with a workspace)
    step     bca_step_attend, every request's cached step (split last round and
             chunk merge included)
    dq       bca_step_attend_dq (e4m3 cache expanded once, then the bf16 kernel)
    q8       bca_step_attend_q8 (e4m3 Q x e4m3 K for the cached keys)
    qkv      bca_qkv_project on the workload's target rows (model width heads x 128)

Every launch is enqueued behind a GPU-busy lead (a spin kernel of
``LEAD_CYCLES``), so the CUDA events around it bracket device time only; the
median over ``reps`` timed calls is printed after one untimed call.  The inputs
are the seeded synthetic tensors of ``workloads`` (layer 0; cached-step inputs of
step 1).  Raises if the library's device status reports an error.
"""
from __future__ import annotations

import statistics
import sys

LEAD_CYCLES = 2_000_000
CASES = ("store", "prefill", "step", "dq", "q8", "qkv")


def _timed(fn, reps: int) -> float:
    import torch
    fn()
    torch.cuda.synchronize()
    ev = []
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda._sleep(LEAD_CYCLES)
        a.record()
        fn()
        b.record()
        ev.append((a, b))
    torch.cuda.synchronize()
    return statistics.median(a.elapsed_time(b) for a, b in ev)


def run(case: str, index: int, reps: int) -> str:
    if case not in CASES:
        raise ValueError(f"unknown case {case!r} (one of {', '.join(CASES)})")
    import torch

    from . import KVSlot, kv_store, kv_store_batch, prefill, qkv_project, step_attend, \
        step_attend_dq, step_attend_q8, step_dq_scratch, step_q8_scratch, step_workspace
    from . import workloads as W

    dev = torch.device("cuda:0")
    wl = W.workload(index)
    H = wl.heads
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    ws = step_workspace(dev)

    def cached_inputs():
        slots = []
        for i, r in enumerate(wl.requests):
            _, k0, v0 = W.qkv(wl, 0, 0, i, dev)
            s = KVSlot(max(r.prefix, 1), H, wl.kv_dtype, device=dev)
            kv_store(k0, v0, r.prefix, s, epoch=1)
            slots.append(s)
            del k0, v0
        per = [W.qkv(wl, 0, 1, i, dev) for i in range(len(wl.requests))]
        q, k, v = (torch.cat([x[j] for x in per]) for j in range(3))
        cu = [0]
        for r in wl.requests:
            cu.append(cu[-1] + r.target)
        return slots, q, k, v, cu

    step_flops = sum(4.0 * 128 * H * r.target * (r.prefix + r.target) for r in wl.requests)
    if case == "store":
        dt = {"bf16": 4, "fp8_v": 3, "fp8": 2}[wl.kv_dtype]  # bytes read + written per element
        items = []
        for i, r in enumerate(wl.requests):
            _, k0, v0 = W.qkv(wl, 0, 0, i, dev)
            items.append((k0, v0, r.prefix, KVSlot(max(r.prefix, 1), H, wl.kv_dtype, device=dev)))
        epoch = [0]

        def fn():
            epoch[0] += 1
            kv_store_batch(items, epoch[0], dev_status=status)
        ms = _timed(fn, reps)
        alg = sum(r.prefix * H * 128 * (4 + dt) for r in wl.requests)
        out = f"store workload {index}: {ms:.4f} ms, {alg / ms / 1e6:.1f} GB/s algorithmic"
    elif case == "prefill":
        r = wl.requests[0]
        q, k, v = W.qkv(wl, 0, 0, 0, dev)
        o = torch.empty_like(q)
        ms = _timed(lambda: prefill(q, k, v, o, r.offsets, wl.scale, dev_status=status,
                                    workspace=ws), reps)
        tot = cum = 0
        for bl in r.blocks:
            cum += bl
            tot += bl * cum
        out = f"prefill workload {index}: {ms:.4f} ms, {4.0 * 128 * H * tot / ms / 1e9:.1f} TFLOP/s"
    elif case in ("step", "dq", "q8"):
        slots, q, k, v, cu = cached_inputs()
        o = torch.empty_like(q)
        if case == "step":
            fn = lambda: step_attend(q, k, v, o, cu, slots, wl.scale, workspace=ws,  # noqa: E731
                                     dev_status=status)
        elif case == "dq":
            sc = step_dq_scratch(slots, dev)
            fn = lambda: step_attend_dq(q, k, v, o, cu, slots, wl.scale, dq_scratch=sc,  # noqa: E731
                                        workspace=ws, dev_status=status)
        else:
            sc = step_q8_scratch(q.shape[0], len(slots), H, dev)
            fn = lambda: step_attend_q8(q, k, v, o, cu, slots, wl.scale, q8_scratch=sc,  # noqa: E731
                                        workspace=ws, dev_status=status)
        ms = _timed(fn, reps)
        out = f"{case} workload {index}: {ms:.4f} ms, {step_flops / ms / 1e9:.1f} TFLOP/s"
    else:  # qkv
        T = sum(r.target for r in wl.requests)
        D = H * 128
        x = W.randn_bf16((T, D), 1, dev)
        w = (W.randn_bf16((3 * D, D), 2, dev).float() * D ** -0.5).to(torch.bfloat16)
        g = torch.ones(128, device=dev)
        c, s = torch.ones(T, 64, device=dev), torch.zeros(T, 64, device=dev)
        q, k, v = (torch.empty(T, H, 128, dtype=torch.bfloat16, device=dev) for _ in range(3))
        ms = _timed(lambda: qkv_project(x, w, q, k, v, g, g, c, s, 1e-6, dev_status=status), reps)
        out = f"qkv workload {index}: {ms:.4f} ms, {2.0 * T * D * 3 * D / ms / 1e9:.1f} TFLOP/s"
    torch.cuda.synchronize()
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())} ({case})")
    return out


def main(argv=None) -> int:
    argv = sys.argv[1:] if argv is None else argv
    if not argv:
        print(__doc__)
        return 2
    case = argv[0]
    index = int(argv[1]) if len(argv) > 1 else 1
    reps = int(argv[2]) if len(argv) > 2 else 5
    print(run(case, index, reps), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
