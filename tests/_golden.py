"""Reader of the hand-derived worked example in tests/golden/bilinear_2x2_worked.txt:
inputs and expected outputs for Cg = 4 channels (channel c holds c+1 times the base
image), grad_out = 1."""
import os

import numpy as np

PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "bilinear_2x2_worked.txt")
BASE = np.array([[1.0, 2.0], [3.0, 4.0]])
CG = 4
GEOMETRY = dict(N=1, H=2, W=2, G=1, Cg=CG, kh=1, kw=1, sh=1, sw=1, ph=0, pw=0, dh=1, dw=1, offset_scale=1.0,
                remove_center=0, P=8)


def load():
    rows, gv = [], None
    for line in open(PATH):
        if line.startswith("pixel"):
            left, right = line.split("|")
            ho, wo, dx, dy, m = left.split()[1:]
            rows.append((int(ho), int(wo), float(dx), float(dy), float(m), [float(t) for t in right.split()]))
        elif line.startswith("grad_value"):
            gv = np.array([float(t) for t in line.split()[1:]]).reshape(2, 2)
    scale = np.arange(1, CG + 1, dtype=np.float64)
    value = (BASE[:, :, None] * scale).reshape(1, 2, 2, CG)
    om = np.zeros((1, 2, 2, 8))
    y = np.zeros((1, 2, 2, CG))
    gom = np.zeros((1, 2, 2, 8))
    for ho, wo, dx, dy, m, (yb, dm, ddx, ddy) in rows:
        om[0, ho, wo, :3] = (dx, dy, m)
        y[0, ho, wo] = yb * scale
        gom[0, ho, wo, :3] = (ddx * scale.sum(), ddy * scale.sum(), dm * scale.sum())
    grad_value = np.repeat(gv[:, :, None], CG, axis=2).reshape(1, 2, 2, CG)
    return dict(value=value, offset_mask=om, grad_out=np.ones((1, 2, 2, CG)), y=y, grad_offset_mask=gom,
                grad_value=grad_value)
