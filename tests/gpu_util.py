"""Helpers for the GPU tests: move seeded inputs to the device and run the C ABI."""
import numpy as np
import torch

import e2ttt_inputs as gen


def dev(x, dtype=torch.float32):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to("cuda").to(dtype)


def act_dtype(w):
    return torch.bfloat16 if w.act == gen.BF16 else torch.float32


def host(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def device_inputs(w, x, zero_m0_as_none=False):
    ad = act_dtype(w)
    d = dict(q=dev(x["q"], ad), k=dev(x["k"], ad), v=dev(x["v"], ad), lr=dev(x["lr"]),
             mom=dev(x["mom"]), decay=dev(x["decay"]), W0=dev(x["W0"]),
             M0=None if zero_m0_as_none else dev(x["M0"]), dout=dev(x["dout"], ad))
    return d


def run_fwd(E, w, d, save=False, ws=None):
    torch.cuda.synchronize()
    out, W_end, M_end, saved = E.chunk_scan_fwd(d["q"], d["k"], d["v"], d["lr"], d["mom"],
                                                d["decay"], d["W0"], d["M0"], C=w.C, d_h=w.d_h,
                                                kind=w.kind, loss=w.loss, save_states=save, ws=ws)
    torch.cuda.synchronize()
    return out, W_end, M_end, saved


def rel(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / nb) if nb > 0 else float(np.linalg.norm(a - b))
