"""The oracle's version of a whole workload: offline preparation on the full
tensors and the runtime path on a chosen set of token rows.  Calls only
``oracle``; the inputs come from the seeded generators."""
from __future__ import annotations

import numpy as np

import oracle


def prepare(w, inp, granularity="per_token"):
    sites = {}
    for site in w.sites:
        st = {"norm": site.norm, "s": None, "s64": None}
        g, b = inp.gamma[site.name], inp.beta[site.name]
        if site.smoothed:
            am = oracle.calibrate_absmax(inp.x_cal[site.name], site.norm, g, b, w.eps)
            Ws = [inp.W[l.name] for l in w.linears_of(site.name)]
            s, s64 = oracle.smooth_scales(am, Ws, w.alpha, w.clamp_eps)
            gf, bf = oracle.fold_norm(s, g, b)
            st.update(act_max=am, s=s, s64=s64, gamma_f=gf, beta_f=bf)
        else:
            st.update(gamma_f=g, beta_f=b)
        st["static_absmax"] = None
        if granularity == "per_tensor_static" and site.smoothed and site.calibrated:
            yc, _, _ = oracle.norm(inp.x_cal[site.name], site.norm, st["gamma_f"], st["beta_f"],
                                   w.eps)
            st["static_absmax"] = oracle.absmax_all(yc)
        sites[site.name] = st
    lins = {}
    for lin in w.linears:
        if granularity == "per_token":
            Wq, ws = oracle.quantize_weights(inp.W[lin.name], sites[lin.site]["s"])
        else:
            Wq, step = oracle.quantize_weights_per_tensor(inp.W[lin.name], sites[lin.site]["s"])
            ws = np.full(lin.N, step, np.float32)
        lins[lin.name] = {"Wq": Wq, "w_scale": ws}
    return {"sites": sites, "linears": lins, "granularity": granularity}


def forward_rows(w, prep, inp, rows):
    """Runtime path for the token rows `rows`: per site (Xq, x_scale), per
    Linear (acc, o32, out bf16 bits)."""
    res = {"sites": {}, "linears": {}}
    for site in w.sites:
        src = next((l.source for l in w.linears if l.site == site.name and l.source), None)
        if src:
            x = res["linears"][src]["out"]
            if site.act == "silu_mul":  # h = SiLU(gate) * up, stored in bf16
                _, x = oracle.silu_mul(x)
        else:
            x = np.ascontiguousarray(inp.x[site.name][rows])
        st = prep["sites"][site.name]
        if prep.get("granularity", "per_token") == "per_token":
            Xq, xs = oracle.norm_quant(x, site.norm, st["gamma_f"], st["beta_f"], w.eps)
        else:  # per-tensor: `rows` must be the whole tensor for O2
            Xq, step = oracle.norm_quant_per_tensor(x, site.norm, st["gamma_f"], st["beta_f"],
                                                    w.eps, absmax=st["static_absmax"])
            xs = np.full(x.shape[0], step, np.float32)
        res["sites"][site.name] = {"x": x, "Xq": Xq, "xs": xs}
        for lin in w.linears_of(site.name):
            L = prep["linears"][lin.name]
            acc = oracle.gemm_i64(Xq, L["Wq"])
            o32, out = oracle.epilogue(acc, xs, L["w_scale"], lin.relu)
            res["linears"][lin.name] = {"acc": acc, "o32": o32, "out": out}
    return res
