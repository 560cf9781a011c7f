"""Write the golden fixtures of this folder from the fp64 oracle.

    python tests/golden/make_golden.py

The pages this project follows print no worked numeric example of the
selective scan or the state update, so these fixtures are not the pages'
values: they are the oracle's own outputs on seeded inputs, stored so that
any later change to the oracle's arithmetic shows up as a failing test
(tests/test_golden.py) and has to be justified.  Only `oracle` and the input
generator are used here; nothing from the CUDA path.
"""
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
from state_space_model_causal_b200 import inputs as gen  # noqa: E402


def cases():
    """(file name, description, {label: array}) of every fixture."""
    out = []
    s = gen.scan_small(seed=0)
    y, h, _ = oracle.scan(s.x, s.dt, s.A, s.B, s.C, D=s.D, z=s.z, dt_bias=s.dt_bias)
    out.append(("scan_small_seed0.txt",
                "Mamba-1 prefill, config 0 recipe: B=1 L=128 D=64 N=16 fp32, no conv, h0=0, seed 0 "
                "(inputs.scan_small(seed=0)); out[0, d, t] for d in 0..3, t in 0..127 step 9, and the "
                "final state h[0, d, :] for d in 0, 63",
                {"out": y[0, :4, ::9], "h_final": h[0, [0, 63], :]}))
    m2 = gen.ssu_mamba2_inputs(2, 4, 8, 16, io="f32", state="f32", seed=0, tag="golden", with_z=True)
    o, st = oracle.ssu_mamba2(m2.state, m2.x, m2.dt, m2.A, m2.B, m2.C, D=m2.D, z=m2.z, dt_bias=m2.dt_bias)
    out.append(("ssu_mamba2_seed0.txt",
                "Mamba-2 decode step: B=2 H=4 P=8 N=16 G=1, fp32, seed 0, tag 'golden' "
                "(inputs.ssu_mamba2_inputs(2, 4, 8, 16, io='f32', state='f32', seed=0, tag='golden', "
                "with_z=True)); out[b, h, :] for (b, h) = (0, 0), (1, 3), and the new state [1, 2, 5, :]",
                {"out": np.stack([o[0, 0], o[1, 3]]), "state": st[1, 2, 5][None]}))
    p2 = gen.scan_m2_inputs(1, 2, 8, 64, 40, io="f32", seed=0, tag="golden", h0=True)
    y2, h2 = oracle.scan_mamba2(p2.x, p2.dt, p2.A, p2.B, p2.C, D=p2.D, z=p2.z, dt_bias=p2.dt_bias, h0=p2.h0)
    out.append(("scan_mamba2_seed0.txt",
                "Mamba-2-layout prefill: B=1 H=2 P=8 N=64 L=40 fp32, seed 0, tag 'golden', h0 given "
                "(inputs.scan_m2_inputs(1, 2, 8, 64, 40, io='f32', seed=0, tag='golden', h0=True)); "
                "out[0, h, p, :] for (h, p) = (0, 0), (1, 7), and the final state [0, 1, 3, :8]",
                {"out": np.stack([y2[0, 0, 0], y2[0, 1, 7]]), "h_final": h2[0, 1, 3, :8][None]}))
    g = gen.gated_conv_inputs(2, 24, 8, 3, io="f32", seed=0, tag="golden", conv_state=True)
    yg, csg = oracle.gated_conv1d(g.x, g.bg, g.cg, g.weight, bias=g.bias, conv_state=g.conv_state)
    out.append(("gated_conv_seed0.txt",
                "double-gated short conv: B=2 L=24 D=8 W=3 fp32, seed 0, tag 'golden', incoming conv state "
                "(inputs.gated_conv_inputs(2, 24, 8, 3, io='f32', seed=0, tag='golden', conv_state=True)); "
                "out[b, d, :] for (b, d) = (0, 0), (1, 7), and the outgoing conv state [1, 3, :]",
                {"out": np.stack([yg[0, 0], yg[1, 7]]), "conv_state": csg[1, 3][None]}))
    return out


def render(desc, arrays):
    lines = ["# written by tests/golden/make_golden.py from the fp64 oracle (not the pages' values)",
             f"# {desc}"]
    for label, a in arrays.items():
        a = np.atleast_2d(np.asarray(a, dtype=np.float64))
        lines.append(f"[{label}] {a.shape[0]} x {a.shape[1]}")
        for row in a:
            lines.append(" ".join(repr(float(v)) for v in row))
    return "\n".join(lines) + "\n"


def parse(text):
    arrays, label, rows = {}, None, []
    for ln in text.splitlines():
        if not ln or ln.startswith("#"):
            continue
        if ln.startswith("["):
            if label:
                arrays[label] = np.array(rows)
            label, rows = ln[1:ln.index("]")], []
        else:
            rows.append([float(v) for v in ln.split()])
    if label:
        arrays[label] = np.array(rows)
    return arrays


if __name__ == "__main__":
    for name, desc, arrays in cases():
        with open(os.path.join(HERE, name), "w") as f:
            f.write(render(desc, arrays))
        print("wrote", name)
