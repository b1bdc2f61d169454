"""Helpers shared by the GPU parity tests (not a test module)."""
import numpy as np
import torch

import oracle.ref as ref
import synth

TOL = {"f32": 1e-5, "bf16": 2e-2}   # max|gpu - ref| / max|ref|, per output tensor


def rel_err(gpu, ref_):
    g = np.asarray(gpu, dtype=np.float64)
    r = np.asarray(ref_, dtype=np.float64)
    den = np.max(np.abs(r))
    num = np.max(np.abs(g - r))
    return float(num / den) if den > 0 else float(num)


def to64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def gpu_run(w: synth.Workload, inputs=None):
    """Forward then backward through the library on cuda:0. Returns CPU
    inputs and the GPU outputs (as torch tensors on the device)."""
    import scaled_dot_product_saving_b200 as lib
    q, k, v, do = synth.make_inputs(w) if inputs is None else inputs
    dev = torch.device("cuda:0")
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    o, lse = lib.attn_fwd(qd, kd, vd, causal=w.causal, scale=w.scale)
    dq, dk, dv = lib.attn_bwd(qd, kd, vd, o, dod, lse, causal=w.causal, scale=w.scale)
    torch.cuda.synchronize()
    assert lib.attn_get_device_error() == 0
    return (q, k, v, do), (o, lse, dq, dk, dv)


def full_compare(w: synth.Workload):
    """Every element of O, LSE, dQ, dK, dV against the float64 oracle."""
    (q, k, v, do), outs = gpu_run(w)
    Q, K, V, dO = (t.to(torch.float64).numpy() for t in (q, k, v, do))
    O, lse = ref.attention_forward(Q, K, V, w.causal, w.scale)
    dQ, dK, dV = ref.attention_backward(Q, K, V, dO, w.causal, w.scale)
    errs = {}
    for name, g, r in zip(("O", "LSE", "dQ", "dK", "dV"), outs, (O, lse, dQ, dK, dV)):
        assert tuple(g.shape) == r.shape, name
        errs[name] = rel_err(to64(g), r)
    return errs


def sampled_compare(w: synth.Workload, heads, n_rows=12, seed=0):
    """Selected rows of a few heads against the oracle, plus invariants over
    every head. Returns (errors, invariant errors)."""
    (q, k, v, do), (o, lse, dq, dk, dv) = gpu_run(w)
    rng = np.random.default_rng(seed)
    errs = {name: 0.0 for name in ("O", "LSE", "dQ", "dK", "dV")}
    for (b, h) in heads:
        qr = sorted(set([0, 1, 127, 128, w.n // 2, w.n - 1] +
                        list(rng.integers(0, w.n, n_rows))))
        kr = sorted(set([0, 1, 127, 128, w.m // 2, w.m - 1] +
                        list(rng.integers(0, w.m, n_rows))))
        qr = [i for i in qr if i < w.n]
        kr = [j for j in kr if j < w.m]
        Qh, Kh, Vh, dOh = (t[b, h].to(torch.float64).numpy() for t in (q, k, v, do))
        O_s, lse_s, dQ_s, dK_s, dV_s = ref.head_backward_sampled(
            Qh, Kh, Vh, dOh, qr, kr, causal=w.causal, scale=w.scale)
        got = {"O": to64(o[b, h])[qr], "LSE": to64(lse[b, h])[qr], "dQ": to64(dq[b, h])[qr],
               "dK": to64(dk[b, h])[kr], "dV": to64(dv[b, h])[kr]}
        want = {"O": O_s, "LSE": lse_s, "dQ": dQ_s, "dK": dK_s, "dV": dV_s}
        for name in errs:
            errs[name] = max(errs[name], rel_err(got[name], want[name]))
    # Invariants over every head (they hold at any size): the rows of dS sum to
    # zero, so the rows of dK sum to zero; the rows of P sum to one, so the rows
    # of dV sum to the rows of dO.
    dk32 = dk.float()
    dv32 = dv.float()
    do32 = do.to(dv.device).float()
    inv = {}
    sum_dk = dk32.sum(dim=2)
    inv["sum_dK"] = float(sum_dk.abs().max() / (dk32.abs().sum(dim=2).max() + 1e-30))
    sum_dv = dv32.sum(dim=2)
    sum_do = do32.sum(dim=2)
    inv["sum_dV"] = float((sum_dv - sum_do).abs().max() / (dv32.abs().sum(dim=2).max() + 1e-30))
    return errs, inv
