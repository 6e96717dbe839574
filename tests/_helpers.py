"""Test helpers: build streams from workloads, tolerance checks."""
import numpy as np

from workloads import DTYPE_BF16, Workload, make_weights

# Tolerances stated for this path: bf16 inputs with fp32 accumulation:
# max|d| <= 1e-2 * max|ref| and sum|d| / sum|ref| <= 2e-3; fp32 configs: 1e-5 for both.
TOL = {DTYPE_BF16: (1e-2, 2e-3), 1: (1e-5, 1e-5)}

# Step-level tolerance of streams with e4m3 operands (la_config.proj_fp8 /
# attn_fp8) against the oracle's own e4m3 definitions.  e4m3 keeps 3 mantissa
# bits (unit roundoff u = 2^-4, against 2^-8 for bf16).  Where an operand lies
# at a rounding boundary, the bf16-level difference between the GPU's chain and
# the fp64 chain moves its code by one e4m3 step, and every e4m3 rounding of the
# step (operand codes of both projections, q, K, V, P) draws such codes again,
# so the step-level difference is of the order of the bf16 tolerance times the
# number of e4m3 roundings in the chain.  Gate: max|d| <= u * max|ref| and
# sum|d| / sum|ref| <= u / 4.
TOL_E4M3_STEP = (2.0 ** -4, 2.0 ** -6)


def step_tolerance(cfg):
    """The tolerance a finished block is gated at against the oracle's step."""
    if getattr(cfg, "proj_fp8", 0) or getattr(cfg, "attn_fp8", 0):
        return TOL_E4M3_STEP
    return TOL[cfg.dtype]


def errors(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    diff = np.abs(got - ref)
    max_rel = diff.max() / max(np.abs(ref).max(), 1e-300)
    mean_rel = diff.sum() / max(np.abs(ref).sum(), 1e-300)
    return max_rel, mean_rel


def assert_close(got, ref, dtype, what="", tol=None):
    tmax, tmean = TOL[dtype] if tol is None else tol
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, f"{what}: shape {got.shape} vs {ref.shape}"
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    max_rel, mean_rel = errors(got, ref)
    assert max_rel <= tmax and mean_rel <= tmean, (
        f"{what}: max|d|/max|ref| = {max_rel:.3e} (tol {tmax}), sum|d|/sum|ref| = {mean_rel:.3e} (tol {tmean})")
    return max_rel, mean_rel


def torch_weights(W, cfg, device="cuda"):
    import torch
    dt = torch.bfloat16 if cfg.dtype == DTYPE_BF16 else torch.float32
    conv = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to(device=device, dtype=dt)
    out = dict(w_qkv=[conv(w) for w in W.w_qkv], w_out=[conv(w) for w in W.w_out],
               w_in=conv(W.w_in), w_head=conv(W.w_head))
    if getattr(W, "w_ffn1", None) is not None:
        out["w_ffn1"] = [conv(w) for w in W.w_ffn1]
        out["w_ffn2"] = [conv(w) for w in W.w_ffn2]
        out["ada"] = torch.from_numpy(np.ascontiguousarray(W.ada, np.float32)).to(device)
    if getattr(W, "w_qc", None) is not None:
        out["w_qc"] = [conv(w) for w in W.w_qc]
        out["w_kvc"] = [conv(w) for w in W.w_kvc]
        out["w_oc"] = [conv(w) for w in W.w_oc]
    return out


def make_stream(wl: Workload, W=None, cfg=None, capture=False):
    import torch
    from streaming_causal_video_timestep_b200 import LaStream
    cfg = cfg or wl.cfg
    W = W if W is not None else make_weights(wl)
    s = LaStream(cfg, torch_weights(W, cfg))
    if capture:
        s.capture(True)
    s.set_sink(torch.from_numpy(W.sink).cuda())
    return s, W


def to_np(t):
    return t.detach().float().cpu().numpy()
