"""Per-entry-point device timings of the library on the synthetic workloads.

    python -m parallelizable_recurrence_b200.kernel_timings [workload ...]

For each workload (default: all of lm_fwd, lm_train, bidir_masked, rec_only,
rec_only_v0) prints one JSON line with the median device time (CUDA events on
the launching stream, 3 warm-up calls, L2 flushed by a 256 MB write before
every timed call) of:
  - sru_forward and sru_backward, and the GB/s of their algorithmic bytes
    (14 B and 24 B per element, bf16 U and dU; padded positions excluded);
  - where the forward scan applies (v = 0), both forced paths;
  - for bf16-projection workloads, sru_project, sru_project_backward (dX and
    dW separately), sru_project_factored (d' = d/4) and, for unidirectional
    layers, SRU++'s attention producer sru_attention_project (d' = d/4,
    causal) in TFLOP/s, beside torch.matmul (cuBLAS) on the same product.
Inputs come from the seeded generator; nothing here checks numerics (the
tests do).
"""
from __future__ import annotations

import json
import sys

import numpy as np
import torch

import parallelizable_recurrence_b200 as sru
from synthetic import CONFIGS, generate

_FLUSH = None


def _timeit(fn, reps: int = 10, warm: int = 3, flush: bool = True) -> float:
    """Median milliseconds of fn() on the current stream."""
    global _FLUSH
    if _FLUSH is None:
        _FLUSH = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device="cuda")
    for _ in range(warm):
        fn()
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps):
        if flush:
            _FLUSH.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    return float(np.median(ts))


def _bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def _f32(a):
    return None if a is None else torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda()


def time_workload(name: str) -> dict:
    cfg = CONFIGS[name]
    L, B, d, nd = cfg.L, cfg.B, cfg.d, cfg.n_dir
    inp = generate(cfg, u_direct=True, with_grad=True)
    U = _bf16(inp["U"]) if inp["U"].dtype == np.uint16 else _f32(inp["U"])
    x, v, b, c0, dh = _f32(inp["x"]), _f32(inp["v"]), _f32(inp["bias"]), _f32(inp["c0"]), _f32(inp["dh"])
    mask = None if inp["mask"] is None else torch.from_numpy(inp["mask"]).cuda()
    valid = 1.0 if inp["mask"] is None else float((inp["mask"] == 0).mean())
    e = L * B * d * nd
    h = torch.empty(L, B, nd, d, device="cuda")
    cT = torch.empty(B, nd, d, device="cuda")
    flags = sru.SRU_FLAG_V_ZERO if cfg.v_zero else 0
    ws = sru.alloc_workspace(L, B, d, nd == 2, flags | sru.SRU_FLAG_FORCE_SCAN)
    dU = torch.empty(L, B, nd, 3, d, device="cuda", dtype=torch.bfloat16)
    dx = torch.empty(L, B, d, device="cuda")
    dv = torch.empty(nd, 2, d, device="cuda")
    db = torch.empty(nd, 2, d, device="cuda")
    dc0 = torch.empty(B, nd, d, device="cuda")
    out = {"workload": name, "L": L, "B": B, "d": d, "n_dir": nd, "elements": e, "valid_fraction": valid}
    variants = [("default", flags)]
    if cfg.v_zero:
        variants += [("sequential", flags | sru.SRU_FLAG_FORCE_SEQUENTIAL), ("scan", flags | sru.SRU_FLAG_FORCE_SCAN)]
    for tag, fl in variants:
        tf = _timeit(lambda: sru.sru_forward(U, x, v, b, h, cT, c0=c0, mask=mask, bidirectional=nd == 2, flags=fl,
                                             workspace=ws))
        tb = _timeit(lambda: sru.sru_backward(U, x, v, b, dh, ws, dU, dx, dv, db, dc0, c0=c0, mask=mask,
                                              bidirectional=nd == 2, flags=fl))
        out[tag] = {"forward_us": tf * 1e3, "forward_GBs": 14 * e * valid / tf / 1e6,
                    "backward_us": tb * 1e3, "backward_GBs": 24 * e * valid / tb / 1e6}
    if cfg.proj_dtype == "bf16":
        M, N, K = L * B, cfg.N, d
        g = torch.Generator(device="cuda").manual_seed(0)
        X = torch.randn(M, K, device="cuda", generator=g).bfloat16()
        W = (torch.randn(N, K, device="cuda", generator=g) / K ** 0.5).bfloat16()
        Uo = torch.empty(M, N, device="cuda", dtype=torch.bfloat16)
        dUo = torch.randn(M, N, device="cuda", generator=g).bfloat16()
        dX = torch.empty(M, K, device="cuda")
        dW = torch.empty(N, K, device="cuda")
        fl = 2.0 * M * N * K
        t_u = _timeit(lambda: sru.sru_project(X, W, Uo), flush=False)
        t_dx = _timeit(lambda: sru.sru_project_backward(dUo, X, W, dX=dX, accumulate=True), flush=False)
        t_dw = _timeit(lambda: sru.sru_project_backward(dUo, X, W, dW=dW), flush=False)
        t_cu = _timeit(lambda: torch.matmul(X, W.t()), flush=False)
        Kp = K // 4
        Wq = (torch.randn(Kp, K, device="cuda", generator=g) / K ** 0.5).bfloat16()
        Wo = (torch.randn(N, Kp, device="cuda", generator=g) / Kp ** 0.5).bfloat16()
        P = torch.empty(M, Kp, device="cuda", dtype=torch.bfloat16)
        dP = torch.empty_like(P)
        dWq = torch.empty(Kp, K, device="cuda")
        dWo = torch.empty(N, Kp, device="cuda")
        ffl = 2.0 * M * Kp * (K + N)
        t_f = _timeit(lambda: sru.sru_project_factored(X, Wq, Wo, P, Uo), flush=False)
        t_fb = _timeit(lambda: sru.sru_project_factored_backward(dUo, X, Wq, Wo, P, dP, dX=dX, accumulate=True,
                                                                 dWq=dWq, dWo=dWo), flush=False)
        t_att = None
        if nd == 1 and L % 8 == 0:
            Wkv = (torch.randn(2 * Kp, Kp, device="cuda", generator=g) / Kp ** 0.5).bfloat16()
            aws = torch.empty(int(sru.load_library().sru_attention_workspace_bytes(L, B, Kp)), dtype=torch.uint8,
                              device="cuda")
            t_att = _timeit(lambda: sru.sru_attention_project(X, Wq, Wkv, Wo, Uo, L, B, 0.5, workspace=aws),
                            flush=False)
        # attention producer flops: Q, [K|V], U products + per batch row 2 L^2 d' (scores) + 2 L^2 d' (A)
        afl = 2.0 * M * Kp * (K + 2 * Kp + N) + 4.0 * B * L * L * Kp
        out["gemm"] = {"M": M, "N": N, "K": K,
                       "project_us": t_u * 1e3, "project_TFs": fl / t_u / 1e9,
                       "dX_us": t_dx * 1e3, "dX_TFs": fl / t_dx / 1e9,
                       "dW_us": t_dw * 1e3, "dW_TFs": fl / t_dw / 1e9,
                       "cublas_project_TFs": fl / t_cu / 1e9,
                       "factored_Kp": Kp, "factored_us": t_f * 1e3, "factored_TFs": ffl / t_f / 1e9,
                       "factored_backward_us": t_fb * 1e3, "factored_backward_TFs": 2 * ffl / t_fb / 1e9}
        if t_att is not None:
            out["gemm"].update(attention_us=t_att * 1e3, attention_TFs=afl / t_att / 1e9)
    status = sru.sru_sync_status()
    if status != 0:
        raise RuntimeError(f"device status {status}")
    return out


def main(argv=None):
    names = (argv if argv is not None else sys.argv[1:]) or ["lm_fwd", "lm_train", "bidir_masked", "rec_only",
                                                             "rec_only_v0"]
    sru.load_library()
    for n in names:
        print(json.dumps(time_workload(n)), flush=True)
        torch.cuda.empty_cache()


if __name__ == "__main__":
    main()
