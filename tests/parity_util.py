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
    kl = w.key_len()
    kl_t = None if kl is None else torch.tensor(kl, dtype=torch.int32, device=dev)
    o, lse = lib.attn_fwd(qd, kd, vd, causal=w.causal, scale=w.scale, key_len=kl_t)
    dq, dk, dv = lib.attn_bwd(qd, kd, vd, o, dod, lse, causal=w.causal, scale=w.scale,
                              key_len=kl_t)
    torch.cuda.synchronize()
    assert lib.attn_get_device_error() == 0
    return (q, k, v, do), (o, lse, dq, dk, dv)


def full_compare(w: synth.Workload):
    """Every element of O, LSE, dQ, dK, dV against the float64 oracle."""
    (q, k, v, do), outs = gpu_run(w)
    Q, K, V, dO = (t.to(torch.float64).numpy() for t in (q, k, v, do))
    kl = w.key_len()
    O, lse = ref.attention_forward(Q, K, V, w.causal, w.scale, key_len=kl)
    dQ, dK, dV = ref.attention_backward(Q, K, V, dO, w.causal, w.scale, key_len=kl)
    errs = {}
    for name, g, r in zip(("O", "LSE", "dQ", "dK", "dV"), outs, (O, lse, dQ, dK, dV)):
        assert tuple(g.shape) == r.shape, name
        errs[name] = rel_err(to64(g), r)
    return errs


def heads_compare(w: synth.Workload, heads):
    """Every element of the selected (batch, head) problems against the oracle,
    plus invariants over every head. Returns (errors, invariant errors); each
    error is max|gpu - ref| / max|ref| over one head, the worst head kept."""
    (q, k, v, do), (o, lse, dq, dk, dv) = gpu_run(w)
    errs = {name: 0.0 for name in ("O", "LSE", "dQ", "dK", "dV")}
    for (b, h) in heads:
        Qh, Kh, Vh, dOh = (t[b, h].to(torch.float64).numpy() for t in (q, k, v, do))
        L = None if w.key_len() is None else w.key_len()[b]
        O_r, lse_r = ref.head_forward(Qh, Kh, Vh, w.causal, w.scale, key_len=L)
        dQ_r, dK_r, dV_r = ref.head_backward(Qh, Kh, Vh, dOh, w.causal, w.scale, key_len=L)
        got = {"O": o[b, h], "LSE": lse[b, h], "dQ": dq[b, h], "dK": dk[b, h], "dV": dv[b, h]}
        want = {"O": O_r, "LSE": lse_r, "dQ": dQ_r, "dK": dK_r, "dV": dV_r}
        for name in errs:
            errs[name] = max(errs[name], rel_err(to64(got[name]), want[name]))
    # Invariants over every head (they hold at any size): the rows of dS sum to
    # zero, so the rows of dK sum to zero; the rows of P sum to one, so the rows
    # of dV sum to the rows of dO.
    dk32, dv32, do32 = dk.float(), dv.float(), do.to(dv.device).float()
    inv = {
        "sum_dK": float(dk32.sum(dim=2).abs().max() / (dk32.abs().sum(dim=2).max() + 1e-30)),
        "sum_dV": float((dv32.sum(dim=2) - do32.sum(dim=2)).abs().max()
                        / (dv32.abs().sum(dim=2).max() + 1e-30)),
    }
    return errs, inv
