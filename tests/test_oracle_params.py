"""Shape pin: the weight shapes the oracle reads (per-head query down-projection
d -> d_I, shared key hidden -> d_I, hidden -> Hq gate; one W_phi [r, d] per
layer and one gate vector per query head) reproduce the parameter overhead the
"IndexMem" technical summary prints in §4 (Efficiency): ~20M indexer and ~0.5M
memory parameters for an 8B model. A query projection from the hidden state,
or one W_phi per KV head, would miss by an order of magnitude."""
import os

from oracle import indexmem_oracle as om

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "param_overhead.txt")


def _read():
    vals, models = {}, []
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        parts = line.split()
        if parts[0] == "model":
            models.append((parts[1],) + tuple(int(x) for x in parts[2:]))
        else:
            vals[parts[0]] = float(parts[1])
    return vals, models


def test_parameter_overhead_matches_pages():
    vals, models = _read()
    tol = vals["tolerance"]
    assert models
    for name, layers, hidden, hq, hd in models:
        idx, mem = om.parameter_counts(hidden, hq, hd, int(vals["idx_dim"]),
                                       int(vals["mem_r"]), layers)
        assert abs(idx / vals["indexer_params"] - 1) <= tol, (name, idx)
        assert abs(mem / vals["memory_params"] - 1) <= tol, (name, mem)


def test_alternative_readings_miss_the_figures():
    vals, models = _read()
    _, layers, hidden, hq, hd = models[0]
    dI, r = int(vals["idx_dim"]), int(vals["mem_r"])
    # queries projected from the hidden state per head
    idx_from_hidden = (hq * hidden * dI + hidden * dI + hidden * hq) * layers
    assert idx_from_hidden / vals["indexer_params"] > 5
    # one W_phi per KV head (8 KV heads)
    mem_per_kv = (8 * r * hd + hq * hd) * layers
    assert mem_per_kv / vals["memory_params"] > 3
