"""Host-side checks of the interaction-layer workloads of bench.py: the layer's shapes close
on themselves (its output has the input's irreps, so layers stack), and the flop and byte
counts used for the roofline agree with the oracle's instruction rule."""
import pytest

import bench
import synth
from oracle.block import GateSpec, linear_instructions, linear_weight_count
from oracle.irreps import Irreps


@pytest.mark.parametrize("base", ["c2", "c4"])
def test_layer_shapes_stack(base):
    spec = synth.CONFIGS[base]
    mul = int(spec.irreps_in.split("x")[0])
    mid, gate_args = bench.layer_shapes(mul)
    g = GateSpec(*gate_args)
    assert g.in_dim == Irreps(mid).dim
    assert g.out_dim == Irreps(spec.irreps_in).dim
    # every gated channel has a gate, and the convolution's output reaches every block of mid
    assert {(l, p) for _, l, p in Irreps(mid).blocks} <= {(l, p) for _, l, p in Irreps(spec.irreps_out).blocks}
    assert len(linear_instructions(spec.irreps_out, mid)) == len(Irreps(mid).blocks)


@pytest.mark.parametrize("ir_in,ir_out", [("32x0e+32x1o+32x2e", "32x0e+32x1o+32x2e"),
                                          ("32x0e+32x1e+32x1o+32x2e+32x2o", "32x0e+64x0e+32x1o+32x2e"),
                                          ("4x0e+12x0e+8x1o+20x3o", "36x0e+8x1o+4x1o+16x3o+8x2e")])
def test_linear_flops_follow_the_instruction_rule(ir_in, ir_out):
    a, b = Irreps(ir_in), Irreps(ir_out)
    want = sum(2 * 7 * (2 * a.blocks[i][1] + 1) * a.blocks[i][0] * b.blocks[o][0]
               for i, o in linear_instructions(ir_in, ir_out))
    assert bench.linear_flops(ir_in, ir_out, 7) == want


def test_layer_node_bytes_count_each_array_once():
    from equivariant_tensor_product_b200 import build
    build.build()
    import equivariant_tensor_product_b200 as tp
    ir_in, ir_out = "32x0e+32x1e+32x1o+32x2e+32x2o", "32x0e+64x0e+32x1o+32x2e"
    lin = tp.Linear(ir_in, ir_out)
    N = 10
    nw = linear_weight_count(ir_in, ir_out)
    assert bench.layer_node_bytes(lin, N, False) == 4 * N * (Irreps(ir_in).dim + Irreps(ir_out).dim) + 4 * nw
    # backward: x and gy read, gx written, W read and gW written
    assert bench.layer_node_bytes(lin, N, True) == 4 * N * (2 * Irreps(ir_in).dim + Irreps(ir_out).dim) + 8 * nw


@pytest.mark.parametrize("base", ["c2", "c3"])
def test_radial_counts_match_the_plan(base):
    """The fused-radial workload counts W_r's width as the plan's weights per edge, and its
    flops are the plain convolution's plus 2 H nw per edge (forward) and three such products
    (backward: projection, gh, gW_r); the edge stream is the hidden row, not the weights."""
    spec = synth.CONFIGS[base]
    N, E, H = 100, 1000, 64
    fb, bb, ff, bf, nw = bench.radial_counts(spec, N, E, H)
    assert nw == synth.n_edge_weights(spec)
    assert ff == bench.fwd_flops(spec, E) + 2 * E * H * nw
    assert bf == bench.bwd_flops(spec, E, False) + 6 * E * H * nw
    in_dim, out_dim = synth.irreps_dim(spec.irreps_in), synth.irreps_dim(spec.irreps_out)
    assert fb == bench.fwd_bytes(N, E, in_dim, out_dim, nw) - E * 4 * nw + E * 4 * H + 4 * H * nw
