"""The synthetic workload generators: graph shapes the configurations state, and the
cell-order relabelling (same workload, spatially ordered labels) used for the labelled
locality variant of the benchmark."""
import numpy as np

import synth
from oracle import OraclePlan, forward


def test_c2_graph_has_exactly_46080_edges_and_valid_csr():
    d = synth.make_inputs("c2", with_gy=False)
    rowptr, src = d["rowptr"], d["src"]
    assert len(rowptr) == 1537 and rowptr[-1] == 46080 == len(src)
    assert np.all(np.diff(rowptr) >= 0)
    assert src.min() >= 0 and src.max() < 1536
    # receiver-sorted CSR: dst is non-decreasing and matches rowptr
    assert np.array_equal(np.repeat(np.arange(1536), np.diff(rowptr)), d["dst"])


def test_cell_sorted_is_a_relabelling_of_the_same_workload():
    d = synth.make_inputs("c2", 192)
    e = synth.cell_sorted(d)
    assert e["info"]["order"] == "cell-sorted"
    N = len(d["rowptr"]) - 1
    assert len(e["src"]) == len(d["src"]) and len(e["rowptr"]) == N + 1
    assert np.array_equal(np.repeat(np.arange(N), np.diff(e["rowptr"])), e["dst"])
    # recover the label map from the node features (rows are distinct random vectors)
    lookup = {d["x"][k].tobytes(): k for k in range(N)}
    perm = np.array([lookup[e["x"][k].tobytes()] for k in range(N)])
    assert sorted(perm.tolist()) == list(range(N))
    spec = d["spec"]
    op = OraclePlan(spec.irreps_in, spec.irreps_sh, spec.irreps_out, spec.paths, "uvu")
    y0 = np.asarray(forward(op, d["rowptr"], d["src"], d["x"], d["vec"], w=d["w"]))
    y1 = np.asarray(forward(op, e["rowptr"], e["src"], e["x"], e["vec"], w=e["w"]))
    np.testing.assert_allclose(y1, y0[perm], rtol=0, atol=1e-12)
    # spatial labels: senders sit closer to their receivers in label space
    gap = lambda g: np.abs(g["src"].astype(np.int64) - g["dst"]).mean()
    assert gap(e) < gap(d)


def test_radial_hidden_inputs_are_seeded_and_shaped():
    d = synth.make_inputs("c1")
    h, Wr = synth.radial_hidden(d)
    h2, Wr2 = synth.radial_hidden(synth.make_inputs("c1"))
    H = d["spec"].mlp_hidden[-1]
    assert h.shape == (len(d["src"]), H) and Wr.shape == (H, d["w"].shape[1])
    assert h.dtype == np.float32 and Wr.dtype == np.float32
    assert np.array_equal(h, h2) and np.array_equal(Wr, Wr2)
    assert np.all(np.isfinite(h)) and np.abs(h).max() > 0
