"""Fixtures under tests/golden/: numbers printed on the pages (cited in the
fixture) and oracle regression values written by a committed script."""
import os

import numpy as np

import oracle
from up_projection_b200 import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _kv(name):
    d = {}
    for line in open(os.path.join(GOLDEN, name)):
        if line.startswith("#") or not line.strip():
            continue
        k, v = line.split(None, 1)
        d.setdefault(k, []).append(v.split())
    return d


def test_astrai_pair_bytes_match_the_page():
    import bench
    d = _kv("astrai_pair_bytes.txt")
    N, K = int(d["N"][0][0]), int(d["K"][0][0])
    # weight bytes of one call = decode_bytes minus the X and H terms
    pair = bench.decode_bytes(1, K, N) - 2 * (K + N)
    assert pair / 2 ** 20 == float(d["pair_MB"][0][0])          # 40.5 (MiB)
    bw = pair / (float(d["time_us"][0][0]) * 1e-6) / 1e12
    assert abs(bw - float(d["bw_TBs"][0][0])) < 0.05            # ~3.1 TB/s


def test_tiny_oracle_regression():
    d = _kv("tiny_oracle.txt")
    X, Wg, Wu = synth.swiglu_inputs(4, 256, 512, "bf16", seed=0)
    out = oracle.swiglu_fwd(X, Wg, Wu, "bf16")
    assert abs(out["H"].sum() - float(d["sum_H"][0][0])) <= 1e-12
    assert abs(np.abs(out["H"]).sum() - float(d["sum_abs_H"][0][0])) <= 1e-12
    for m, n, v in d["H"]:
        assert out["H"][int(m), int(n)] == float(v)
