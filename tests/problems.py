"""Small seeded problems already in the W8A8 operand format (int8 or soft-edge
codes plus fp32 scales).  Only random draws happen here (synth helpers); the
same arrays feed the oracle and the CUDA path."""
import numpy as np

from quantized_state_space_b200 import synth


def m1_problem(seed, b, L, d, N, G=1, gs=4, *, k_x=4, gate=True, h0=False, bias=False,
               x_format="int8", dt_mean=-4.0, a_lo=0.0):
    rng = np.random.default_rng(seed)
    p = {}
    if x_format == "int8":
        p["x"] = synth.random_codes(rng, (b, d, L))
        p["x_group"] = rng.integers(0, k_x, size=d).astype(np.int32)
        p["x_scale"] = synth.random_scales(rng, k_x, 0.005, 0.05)
    else:
        p["x"] = synth.random_bytes(rng, (b, d, L))
        p["se_scale"] = float(synth.random_scales(rng, 1, 0.01, 0.05)[0])
    p["dt"] = (rng.standard_normal((b, d, L)) * 0.5 + dt_mean).astype(np.float16)
    p["A"] = (-np.exp(rng.uniform(a_lo, np.log(16.0), size=(d, N)))).astype(np.float32)
    p["D"] = rng.standard_normal(d).astype(np.float32)
    p["z"] = rng.standard_normal((b, d, L)).astype(np.float16) if gate else None
    p["B"] = synth.random_codes(rng, (b, G, N, L))
    p["C"] = synth.random_codes(rng, (b, G, N, L))
    p["B_scale"] = synth.random_scales(rng, G * N // gs, 0.005, 0.03)
    p["C_scale"] = synth.random_scales(rng, G * N // gs, 0.005, 0.03)
    p["h0"] = (rng.standard_normal((b, d, N)) * 0.1).astype(np.float32) if h0 else None
    p["dt_bias"] = (rng.standard_normal(d) * 0.1).astype(np.float32) if bias else None
    p["state_group_size"] = gs
    return p


def ssd_problem(seed, b, L, H, P, N, G=1, gs=8, *, k_x=4, gate=False, h0=False, bias=False,
                x_format="int8", dt_mean=-4.0):
    rng = np.random.default_rng(seed)
    p = {}
    if x_format == "int8":
        p["x"] = synth.random_codes(rng, (b, L, H, P))
        head_cluster = rng.integers(0, k_x, size=H)
        p["x_group"] = np.repeat(head_cluster, P).astype(np.int32)
        p["x_scale"] = synth.random_scales(rng, k_x, 0.005, 0.05)
    else:
        p["x"] = synth.random_bytes(rng, (b, L, H, P))
        p["se_scale"] = float(synth.random_scales(rng, 1, 0.01, 0.05)[0])
    p["dt"] = (rng.standard_normal((b, L, H)) * 0.5 + dt_mean).astype(np.float16)
    p["A"] = (-np.exp(rng.uniform(0.0, np.log(16.0), size=H))).astype(np.float32)
    p["D"] = rng.standard_normal(H).astype(np.float32)
    p["z"] = rng.standard_normal((b, L, H, P)).astype(np.float16) if gate else None
    p["B"] = synth.random_codes(rng, (b, L, G, N))
    p["C"] = synth.random_codes(rng, (b, L, G, N))
    p["B_scale"] = synth.random_scales(rng, G * N // gs, 0.005, 0.03)
    p["C_scale"] = synth.random_scales(rng, G * N // gs, 0.005, 0.03)
    p["h0"] = (rng.standard_normal((b, H, P, N)) * 0.1).astype(np.float32) if h0 else None
    p["dt_bias"] = (rng.standard_normal(H) * 0.1).astype(np.float32) if bias else None
    p["state_group_size"] = gs
    return p


def oracle_kwargs(p):
    """Keyword arguments of the oracle's scan functions for a problem dict."""
    kw = dict(D=p["D"], z=p["z"], dt_bias=p["dt_bias"], h0=p.get("h0"))
    if p["x"].dtype == np.uint8:
        kw["se_scale"] = p["se_scale"]
    else:
        kw["x_group"] = p["x_group"]
        kw["x_scale"] = p["x_scale"]
    return kw
