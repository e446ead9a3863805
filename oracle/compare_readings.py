"""How far the oracle's two backward readings sit from their textbook alternatives.

Run: ``python -m oracle.compare_readings [config]`` (default: mid).  Prints, for the
weight gradients and d(combine weight), the relative Frobenius distance between the
reading the layer implements (weight-gradient operands requantised from the MX payloads
the data path holds; d(combine weight) = <G, h^>) and the plain one (operands quantised
from the unquantised bf16 values; <dOut, y>), and the distance of each from the exact,
unquantised gradients.  Test infrastructure: it calls only the oracle and the seeded
input generators.
"""
from __future__ import annotations

import sys

import numpy as np

import synth
from oracle import layer as L


def _rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def main(name: str = "mid") -> None:
    case = synth.CONFIGS[name]
    x, lg, dout = synth.make_x(case), synth.make_logits(case), synth.make_dout(case)
    cache = {}

    def wfn(e):
        if e not in cache:
            cache[e] = synth.expert_weights_f64(case, e)
        return cache[e]
    args = (x, lg, dout, case.k, case.score_fn, case.E, wfn)
    ours = L.backward(*args, want_dx=False)
    plain = L.backward(*args, want_dx=False, plain=True)
    exact = L.backward(*args, want_dx=False, exact=True)

    def stack(r, m):
        return np.concatenate([r["dW"][e][m].ravel() for e in sorted(r["dW"])])
    for m, nm in enumerate(("dW_gate", "dW_up", "dW_down")):
        a, b, c = stack(ours, m), stack(plain, m), stack(exact, m)
        print(f"{name} {nm}: reading vs plain {_rel(a, b):.3e}; vs exact: reading "
              f"{_rel(a, c):.3e}, plain {_rel(b, c):.3e}")
    print(f"{name} d(combine weight): reading vs plain {_rel(ours['dw'], plain['dw']):.3e}; "
          f"vs exact: reading {_rel(ours['dw'], exact['dw']):.3e}, "
          f"plain {_rel(plain['dw'], exact['dw']):.3e}")


if __name__ == "__main__":
    main(sys.argv[1] if len(sys.argv) > 1 else "mid")
