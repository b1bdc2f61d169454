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


def gpu_run(w: synth.Workload, inputs=None, dq_path=None):
    """Forward then backward through the library on cuda:0 (with the calling
    thread's dQ design set to `dq_path` for the call, if given). Returns CPU
    inputs and the GPU outputs (as torch tensors on the device)."""
    import scaled_dot_product_saving_b200 as lib
    q, k, v, do = synth.make_inputs(w) if inputs is None else inputs
    dev = torch.device("cuda:0")
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    kl = w.key_len()
    kl_t = None if kl is None else torch.tensor(kl, dtype=torch.int32, device=dev)
    if dq_path is not None:
        lib.attn_set_dq_path(dq_path)
    try:
        o, lse = lib.attn_fwd(qd, kd, vd, causal=w.causal, scale=w.scale, key_len=kl_t)
        dq, dk, dv = lib.attn_bwd(qd, kd, vd, o, dod, lse, causal=w.causal, scale=w.scale,
                                  key_len=kl_t)
    finally:
        if dq_path is not None:
            lib.attn_set_dq_path(lib.ATTN_DQ_AUTO)
    torch.cuda.synchronize()
    assert lib.attn_get_device_error() == 0
    return (q, k, v, do), (o, lse, dq, dk, dv)


def full_compare(w: synth.Workload, dq_path=None):
    """Every element of O, LSE, dQ, dK, dV against the float64 oracle."""
    (q, k, v, do), outs = gpu_run(w, dq_path=dq_path)
    Q, K, V, dO = (t.to(torch.float64).numpy() for t in (q, k, v, do))
    kl = w.key_len()
    O, lse = ref.attention_forward(Q, K, V, w.causal, w.scale, key_len=kl)
    dQ, dK, dV = ref.attention_backward(Q, K, V, dO, w.causal, w.scale, key_len=kl)
    errs = {}
    for name, g, r in zip(("O", "LSE", "dQ", "dK", "dV"), outs, (O, lse, dQ, dK, dV)):
        assert tuple(g.shape) == r.shape, name
        errs[name] = rel_err(to64(g), r)
    return errs


def scheduler_heads(w: synth.Workload):
    """The (batch, head) problems that a full-size test compares element by
    element: the first, middle and last head of every head group of the
    tensor-core backward's and forward's schedules (groups of about 256 work
    items: 128 keys per backward item, two 128-row query tiles per forward
    item; when causal the backward merges its last two groups into one), so
    that every group is checked. Heads are numbered b*H + h."""
    BH = w.B * w.H
    picked = set()
    num_kt = -(-w.m // 128)
    num_pairs = -(-(-(-w.n // 128)) // 2)
    for items_per_head, merge_last in ((num_kt, w.causal), (num_pairs, False)):
        hg = max(1, min(BH, 256 // items_per_head))
        starts = list(range(0, BH, hg))
        if merge_last and len(starts) >= 2:
            starts.pop()
        for i, g0 in enumerate(starts):
            last = (starts[i + 1] if i + 1 < len(starts) else BH) - 1
            picked.update({g0, (g0 + last) // 2, last})
    return [(x // w.H, x % w.H) for x in sorted(picked)]


def all_heads(w: synth.Workload):
    return [(b, h) for b in range(w.B) for h in range(w.H)]


def heads_compare(w: synth.Workload, heads, dq_paths=(None,)):
    """Every element of the selected (batch, head) problems against the oracle,
    plus invariants over every head, for each dQ design in `dq_paths` (the
    oracle runs once per head). Returns (errors, invariant errors) for a single
    design, else a dict design -> (errors, invariant errors); each error is
    max|gpu - ref| / max|ref| over one head, the worst head kept."""
    inputs = synth.make_inputs(w)
    q, k, v, do = inputs
    runs = {p: gpu_run(w, inputs, dq_path=p)[1] for p in dq_paths}
    errs = {p: {name: 0.0 for name in ("O", "LSE", "dQ", "dK", "dV")} for p in dq_paths}
    for (b, h) in heads:
        Qh, Kh, Vh, dOh = (t[b, h].to(torch.float64).numpy() for t in (q, k, v, do))
        L = None if w.key_len() is None else w.key_len()[b]
        O_r, lse_r = ref.head_forward(Qh, Kh, Vh, w.causal, w.scale, key_len=L)
        dQ_r, dK_r, dV_r = ref.head_backward(Qh, Kh, Vh, dOh, w.causal, w.scale, key_len=L)
        want = {"O": O_r, "LSE": lse_r, "dQ": dQ_r, "dK": dK_r, "dV": dV_r}
        for p, (o, lse, dq, dk, dv) in runs.items():
            got = {"O": o[b, h], "LSE": lse[b, h], "dQ": dq[b, h], "dK": dk[b, h], "dV": dv[b, h]}
            for name in errs[p]:
                errs[p][name] = max(errs[p][name], rel_err(to64(got[name]), want[name]))
    # Invariants over every head (they hold at any size): the rows of dS sum to
    # zero, so the rows of dK sum to zero; the rows of P sum to one, so the rows
    # of dV sum to the rows of dO.
    out = {}
    for p, (o, lse, dq, dk, dv) in runs.items():
        dk32, dv32, do32 = dk.float(), dv.float(), do.to(dv.device).float()
        inv = {
            "sum_dK": float(dk32.sum(dim=2).abs().max() / (dk32.abs().sum(dim=2).max() + 1e-30)),
            "sum_dV": float((dv32.sum(dim=2) - do32.sum(dim=2)).abs().max()
                            / (dv32.abs().sum(dim=2).max() + 1e-30)),
        }
        out[p] = (errs[p], inv)
    return out[dq_paths[0]] if len(dq_paths) == 1 else out
