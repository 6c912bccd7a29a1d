"""Calibrate the utility perceptron's output bias b2 for each workload.

TEST INFRASTRUCTURE (input preparation): run once with
``python -m oracle.calibrate``; it writes
``sparse_decode_attention_spkv_b200/inputs/biases.json``, which the workloads read
as an input like any weight.  Only the oracle's fp64 perceptron is evaluated here.

For key head k with target keep rate p_k, b2_k = logit(tau) - Q_{1-p_k}(l_k), where
l_k is the pre-bias logit f(h) - b2 of Eq. (1) of "Self-Pruned Key-Value Attention"
(arXiv 2605.14037) over a calibration draw of hidden states with the data's
distribution (stream T_CAL of the generator).  Then u >= tau (Eq. 2) holds for a
fraction p_k of that draw.
"""
from __future__ import annotations

import json
import math
import sys

import numpy as np

from oracle import spkv_oracle as O
from sparse_decode_attention_spkv_b200.inputs import workloads as W

N_CAL = 4096


def calibrate(wl: W.Workload, n_cal: int = N_CAL) -> dict:
    out = {"b2": [], "keep_target": [], "n_cal": n_cal}
    logit_tau = math.log(wl.tau / (1.0 - wl.tau))
    for layer in range(wl.layers):
        h = wl.calib_h(layer, n_cal)
        raw = O.utility_logits(h, wl.w1(layer), wl.b1(layer), wl.w2(layer), np.zeros(wl.Hkv))
        p = wl.keep_targets(layer)
        b2 = [float(np.float32(logit_tau - np.quantile(raw[:, k], 1.0 - p[k])))
              for k in range(wl.Hkv)]
        out["b2"].append(b2)
        out["keep_target"].append([float(x) for x in p])
    return out


def main(names=None):
    names = names or list(W.WORKLOADS)
    table = dict(W.load_biases())
    for name in names:
        print("calibrating", name, file=sys.stderr)
        table[name] = calibrate(W.WORKLOADS[name])
    with open(W.bias_file(), "w") as f:
        json.dump(table, f, indent=1)


if __name__ == "__main__":
    main(sys.argv[1:])
