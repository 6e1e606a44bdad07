"""Pipeline timelines of the SpMM kernels (a profiling aid, not part of the product path).

Runs problems through ``libnmspmm_trace.so`` (``build.py --trace``: the same
sources compiled with NM_TRACE), whose kernels record, per CTA,
  * SM-clock stamps of every pipeline stage: producer issue, operands landed
    (seen by the MMA warp), MMAs issued, and per tile the epilogue start and end;
  * global-timer stamps (ns, comparable across SMs) at kernel entry, after the
    wait on the previous kernel, after the role loops and at exit.
It reports, per problem, the medians over CTAs of: the MMA warp's wait for
operands, the stage cadence, the load latency (issue to landed), the epilogue
time per tile and the tile period; and, for a sequence captured in one CUDA
graph, the time from the previous kernel's last CTA exit to the first return
from the wait, and the spread of CTA exits.

    python -m structured_sparse_gemm_compress_b200.trace --problems vitb.qkv/2:4,vitb.fc2/2:4 --out t.json

Problems are named like the bench's (``vitb.<layer>/<N:M>`` at T = 12608,
``vitl.<layer>/<N:M>`` at T = 6304) and use the same seeded inputs.  Must run
in a fresh process: the binding loads the trace library instead of the product one.
"""
from __future__ import annotations

import argparse
import json
import os

import numpy as np
import torch

from . import build, inputs

KMAX, KINDS = 64, 7  # slots per kind and kinds per CTA (trace layout of the NM_TRACE build)
P_ISSUE, M_FULL, M_DONE, M_ACCE, E_START, E_END, GT = range(7)


def _problem(name: str):
    pool = inputs.vit_l_fp16() if name.startswith("vitl") else inputs.vit_b_int8()
    for l in pool:
        if f"{l.name}/{l.nm}" == name:
            return l
    raise SystemExit(f"unknown problem {name}")


def _setup(nm, name: str):
    l = _problem(name)
    W, X = l.weight().cuda(), l.activation().cuda()
    s = l.scale().cuda() if l.scaled else None
    h = nm.nm_compress(W, l.N, l.M)
    plan = nm.nm_plan_query(h, l.T, scaled=s is not None)
    nblk = plan["grid"] * (2 if plan["pair"] else 1)
    buf = torch.zeros(nblk * KINDS * KMAX, dtype=torch.int64, device="cuda")
    Y = torch.empty((l.T, l.n_out), dtype=nm.out_dtype(h, s is not None), device="cuda")
    return {"name": name, "h": h, "X": X, "s": s, "Y": Y, "buf": buf, "nblk": nblk, "plan": plan}


def _stage_stats(tr: np.ndarray, pair: bool) -> dict:
    waits, cad, lat, epi, period = [], [], [], [], []
    for b in (range(0, tr.shape[0], 2) if pair else range(tr.shape[0])):  # the issuing CTA of a pair
        P, F, D, ES, EE = tr[b, P_ISSUE], tr[b, M_FULL], tr[b, M_DONE], tr[b, E_START], tr[b, E_END]
        n = int((F > 0).sum())
        for i in range(1, n):
            if F[i] > 0 and D[i - 1] > 0:
                waits.append(F[i] - D[i - 1])
                cad.append(D[i] - D[i - 1])
            if F[i] > 0 and P[i] > 0:
                lat.append(F[i] - P[i])
        ne = int((ES > 0).sum())
        epi += [EE[i] - ES[i] for i in range(ne) if EE[i] > 0]
        if ne > 1:
            period += list(np.diff(ES[:ne]))
    med = lambda a: int(np.median(a)) if len(a) else None
    return {"mma_wait_cycles": med(waits), "stage_cadence_cycles": med(cad), "load_latency_cycles": med(lat),
            "epilogue_cycles_per_tile": med(epi), "tile_period_cycles": med(period)}


def run(problems: list[str], raw_out: bool = False) -> dict:
    build.build(trace=True)
    import structured_sparse_gemm_compress_b200 as nm
    if nm._lib is not None:
        raise RuntimeError("the product library is already loaded in this process")
    nm.LIB_PATH = build.TRACE_LIB
    torch.cuda.set_device(0)
    probs = [_setup(nm, n) for n in problems]
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream, capture_error_mode="thread_local"):
        for p in probs:  # the trace buffer is a launch argument: set while capturing each launch
            os.environ["NMSPMM_TRACE_PTR"] = str(p["buf"].data_ptr())
            nm.nm_spmm(p["h"], p["X"], Y=p["Y"], scale=p["s"], stream=stream)
    os.environ.pop("NMSPMM_TRACE_PTR", None)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    for p in probs:
        p["buf"].zero_()
    torch.cuda.synchronize()
    g.replay()
    torch.cuda.synchronize()
    out, prev_exit, base = [], None, None
    for p in probs:
        if nm.nm_device_status(p["h"]) != nm.NM_OK:
            raise RuntimeError(nm.nm_last_error())
        tr = p["buf"].view(p["nblk"], KINDS, KMAX).cpu().numpy()
        gt = tr[:, GT, :4]
        gt = gt[gt[:, 0] > 0]
        base = gt[:, 0].min() if base is None else base
        raw = {f"cta{b}": {k: [int(x) for x in tr[b, i, :24]] for i, k in
                           enumerate(("p_issue", "m_full", "m_done", "m_acce", "e_start", "e_end"))}
               for b in (0, 1) if b < tr.shape[0]}
        for b in (0, 1):
            if b < tr.shape[0]:
                raw[f"cta{b}"]["gt_ns"] = [int(x - base) for x in tr[b, GT, :4]]
                raw[f"cta{b}"]["gt_clk"] = [int(x) for x in tr[b, GT, 4:8]]
        r = {"problem": p["name"], "plan": p["plan"], **_stage_stats(tr, bool(p["plan"]["pair"])),
             "entry_us": round((gt[:, 0].min() - base) / 1e3, 2), "first_wait_return_us": round((gt[:, 1].min() - base) / 1e3, 2),
             "exit_first_us": round((gt[:, 3].min() - base) / 1e3, 2), "exit_last_us": round((gt[:, 3].max() - base) / 1e3, 2)}
        if prev_exit is not None:
            r["prev_last_exit_to_first_wait_return_us"] = round((gt[:, 1].min() - prev_exit) / 1e3, 2)
        if raw_out:
            r["raw_first_ctas"] = raw
        prev_exit = gt[:, 3].max()
        out.append(r)
        p["h"].destroy()
    del g
    return {"problems": out, "note": "cycles: SM clock; us: global timer, origin = first kernel entry"}


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--problems", required=True, help="comma-separated, e.g. vitb.qkv/2:4,vitb.fc2/2:4")
    ap.add_argument("--out", default=None)
    ap.add_argument("--raw", action="store_true", help="also keep the first CTAs' raw stamps (first 24 of each kind)")
    a = ap.parse_args()
    res = run(a.problems.split(","), raw_out=a.raw)
    for r in res["problems"]:
        print(json.dumps({k: v for k, v in r.items() if k != "raw_first_ctas"}))
    if a.out:
        json.dump(res, open(a.out, "w"), indent=1)


if __name__ == "__main__":
    main()
