"""Shared test utilities: error metrics and sampled-head oracle runs."""
import numpy as np
import torch

import oracle

TOL_F32 = 1e-4     # fp32 inputs: max|do|/RMS(o_ref) and state relative Frobenius error
TOL_BF16 = 5e-3    # bf16 inputs, fp32 state and accumulation


def o_err(o_gpu, o_ref) -> float:
    """max |o_gpu - o_ref| / RMS(o_ref) over the whole tensor."""
    o_gpu = np.asarray(o_gpu.detach().float().cpu().double() if torch.is_tensor(o_gpu) else o_gpu)
    o_ref = np.asarray(o_ref, dtype=np.float64)
    rms = np.sqrt(np.mean(o_ref ** 2))
    return float(np.abs(o_gpu - o_ref).max() / rms)


def s_err(s_gpu, s_ref) -> float:
    """||S_gpu - S_ref||_F / ||S_ref||_F."""
    s_gpu = np.asarray(s_gpu.detach().float().cpu().double() if torch.is_tensor(s_gpu) else s_gpu)
    s_ref = np.asarray(s_ref, dtype=np.float64)
    return float(np.linalg.norm(s_gpu - s_ref) / np.linalg.norm(s_ref))


def tol_for(x) -> float:
    return TOL_F32 if x["q"].dtype == torch.float32 and x["alpha"].dtype == torch.float32 else TOL_BF16


def oracle_full(x):
    """Oracle over every (sequence, head) of a prefill input dict (tensors on any device)."""
    cpu = {k: (v.cpu() if torch.is_tensor(v) else v) for k, v in x.items()}
    return oracle.forward(cpu["q"], cpu["k"], cpu["v"], cpu["alpha"], cpu["beta"],
                          s0=cpu.get("s0"), scale=cpu["scale"])


def oracle_heads(x, pairs):
    """Oracle for selected (b, h) pairs only: returns {(b,h): (o [T,dv], S [dk,dv])}."""
    out = {}
    for b, h in pairs:
        sl = lambda t: t[b:b + 1, :, h:h + 1].cpu()
        s0 = None if x.get("s0") is None else x["s0"][b:b + 1, h:h + 1].cpu()
        o, S = oracle.forward(sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(x["alpha"]),
                              x["beta"][b:b + 1, :, h:h + 1].cpu(), s0=s0, scale=x["scale"])
        out[(b, h)] = (o[0, :, 0], S[0, 0])
    return out


def to_device(x, device="cuda"):
    return {k: (v.to(device) if torch.is_tensor(v) else v) for k, v in x.items()}
