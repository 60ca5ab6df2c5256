"""Write the ``closed_form_*.json`` fixtures: worked examples of the PACK3D operator whose
outputs follow in closed form, derived by hand (this script uses only ``math``).

Source of the definition: "Geometry Matters in Packed 3D Attention", abstract --
exact local neighbourhood attention, contiguous 3D block summaries taken after
the rotation, and axial RoPE on true grid coordinates.  The pages print no
worked example, so this one is constructed from that definition.

Set-up.  A line of 4 tokens along one axis (extent 1 on the other two); one
head; window 1 x 1 x 1 (each query sees only itself); blocks of 2 along the
line: block 0 holds coordinates 0, 1 and block 1 holds 2, 3.

Inputs.  Every q and k is the unit vector on the first channel of one rotation
pair of that axis, with frequency theta, so rotated vectors are
(cos(theta c), sin(theta c)) on that pair and q~_i . k~_j = cos(theta (c_j - c_i)).
v_j = (j + 1) on one channel and (j + 1)^2 on another, zero elsewhere.

Derivation.  A query at x sees itself (logit tau, since cos 0 = 1) and the
summary of the one block that does not hold it (the block holding it meets its
window).  The summary key is the mean of the two rotated keys, so its logit is
tau * (cos(theta (c_a - c)) + cos(theta (c_b - c))) / 2 for that block's members
c_a, c_b; the summary value is the mean of their values.  Then
o = (e^s v_self + e^t vbar) / (e^s + e^t) and lse = ln(e^s + e^t), with
tau = 1 / sqrt(d) and no count bias on t.
"""
import json
import math
import os

L = 4  # extent along the chosen axis


def fixture(axis, d, channel, theta, v_channels=(0, 1)):
    """Volume of extent L along ``axis`` (0 = z, 1 = y, 2 = x) and 1 elsewhere.

    q and k are the unit vector on ``channel``, the first member of a rotation
    pair of that axis whose frequency is ``theta``; rotated vectors are then
    (cos(theta c), sin(theta c)) on the pair and q~_i . k~_j = cos(theta (c_j - c_i))."""
    tau = 1.0 / math.sqrt(d)
    unit = [0.0] * d
    unit[channel] = 1.0
    q = [list(unit) for _ in range(L)]
    k = [list(unit) for _ in range(L)]
    v = []
    for j in range(L):
        row = [0.0] * d
        row[v_channels[0]] = float(j + 1)
        row[v_channels[1]] = float((j + 1) ** 2)
        v.append(row)
    blocks = [(0, 1), (2, 3)]
    out, lse = [], []
    for c in range(L):
        other = blocks[1] if c < 2 else blocks[0]
        s = tau * math.cos(0.0)
        t = tau * (math.cos(theta * (other[0] - c)) + math.cos(theta * (other[1] - c))) / 2.0
        vbar = [(v[other[0]][e] + v[other[1]][e]) / 2.0 for e in range(d)]
        es, et = math.exp(s), math.exp(t)
        out.append([(es * v[c][e] + et * vbar[e]) / (es + et) for e in range(d)])
        lse.append(math.log(es + et))
    ext = [1, 1, 1]
    ext[axis] = L
    blk = [1, 1, 1]
    blk[axis] = 2
    coords = []
    for c in range(L):
        cc = [0, 0, 0]
        cc[axis] = c
        coords.append(cc)
    return {
        "source": "Geometry Matters in Packed 3D Attention, abstract (local exact attention, "
                  "block summaries of rotated keys, axial RoPE on grid coordinates); "
                  "worked example derived by hand in make_closed_form.py",
        "shape": {"B": 1, "H": 1, "d": d, "Z": ext[0], "Y": ext[1], "X": ext[2],
                  "window": [1, 1, 1], "block": blk, "rope_base": 100.0},
        "theta": theta, "channel": channel,
        "coords": coords, "q": q, "k": k, "v": v, "out": out, "lse": lse,
    }


CASES = {
    # d = 6: one pair per axis, frequency base^0 = 1; x pair = channels (4, 5).
    "closed_form_x_d6.json": dict(axis=2, d=6, channel=4, theta=1.0),
    # d = 12: two pairs per axis; the second x pair is channels (9, 11) and its
    # frequency is 100^(-2*1/4) = 0.1.
    "closed_form_x_d12_pair1.json": dict(axis=2, d=12, channel=9, theta=0.1),
    # d = 6 along z: the z pair is channels (0, 1); v lives on channels 2, 3.
    "closed_form_z_d6.json": dict(axis=0, d=6, channel=0, theta=1.0, v_channels=(2, 3)),
    # d = 12 along y: first y pair is channels (4, 6), frequency 1.
    "closed_form_y_d12_pair0.json": dict(axis=1, d=12, channel=4, theta=1.0),
}


def main():
    here = os.path.dirname(os.path.abspath(__file__))
    for name, kw in CASES.items():
        with open(os.path.join(here, name), "w") as f:
            json.dump(fixture(**kw), f, indent=1)
            f.write("\n")


if __name__ == "__main__":
    main()
