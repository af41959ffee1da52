"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every symbol
the headers under include/ declare, and rejects bad plans and bad calls with the documented status
before touching the device."""
import ctypes as C
import os
import re

import pytest

import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from equivariant_tensor_product_b200 import build
    build.build()
    from equivariant_tensor_product_b200 import _lib
    return _lib.load()


@pytest.fixture(scope="module")
def tp(lib):
    import equivariant_tensor_product_b200 as tp
    return tp


def _declared_symbols():
    inc = os.path.join(ROOT, "include")
    text = "\n".join(open(os.path.join(inc, f)).read() for f in sorted(os.listdir(inc)) if f.endswith(".h"))
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(tp_[a-z_]+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    names = _declared_symbols()
    assert len(names) >= 24
    for n in names:
        assert hasattr(lib, n), n
    out = os.popen(f"nm -D --defined-only {os.path.join(ROOT, 'equivariant_tensor_product_b200', 'libtp.so')}").read()
    for n in names:
        assert re.search(rf"\bT {n}\b", out), f"{n} not exported as a text symbol"


def test_version_and_status_strings(lib):
    assert b"sm_100a" in lib.tp_version()
    assert lib.tp_status_string(0) == b"ok"
    assert lib.tp_status_string(4) == b"workspace too small"


@pytest.mark.parametrize("name", ["c1", "c2", "c3", "c4", "c5"])
def test_plan_matches_config_sizes(tp, name):
    spec = synth.CONFIGS[name]
    plan = tp.Plan(spec.irreps_in, spec.irreps_sh, spec.irreps_out, spec.paths, spec.mode)
    assert plan.in_dim == synth.irreps_dim(spec.irreps_in)
    assert plan.out_dim == synth.irreps_dim(spec.irreps_out)
    assert plan.n_edge_weights == synth.n_edge_weights(spec)
    if spec.mode == "uvw":
        P, U, V = synth.shared_weight_shape(spec)
        assert plan.n_shared_weights == P * U * V


@pytest.mark.parametrize("args,status", [
    (("4x0e+4x1o", "1x0e+1x1o", "4x0e+4x1o", [(0, 0, 0), (0, 1, 1), (1, 0, 1), (1, 1, 0)]), 0),
    (("4x0e+4x1q", "1x0e+1x1o", "4x0e+4x1o", [(0, 0, 0)]), 1),          # bad parity letter
    (("4x0e+", "1x0e", "4x0e", [(0, 0, 0)]), 1),                           # trailing +
    (("0x0e", "1x0e", "4x0e", [(0, 0, 0)]), 1),                            # zero multiplicity
    (("4x4e", "1x0e", "4x4e", [(0, 0, 0)]), 2),                            # l > 3
    (("4x0e+4x1o", "1x0e+1x1e", "4x0e+4x1o", [(0, 0, 0)]), 1),          # SH parity
    (("4x0e+4x1o", "1x0e+1x1o", "4x0e+4x1o", [(0, 1, 0)]), 1),          # triangle
    (("4x0e+4x1o", "1x0e+1x1o", "4x0e+4x1o", [(1, 1, 1)]), 1),          # parity 1o x 1o -> 1o
    (("4x0e+4x1o", "1x0e+1x1o", "8x0e+8x1o", [(0, 0, 0)]), 1),          # uvu multiplicity
    (("4x0e+4x1o", "1x0e+1x1o", "4x0e+4x1o", [(0, 0, 0)]), 0),          # valid, runtime path table
    (("8x1o+4x0e", "1x0e+1x1o+1x2e", "4x1o+8x2e+8x1o", [(1, 1, 0), (0, 0, 1)]), 1),   # 1o x 0e -> 2e
    (("8x1o+4x0e", "1x0e+1x1o+1x2e", "4x1o+8x2e+8x1o", [(1, 1, 0), (0, 1, 2)]), 1),   # 1o x 1o -> 1o
    (("8x1o+4x0e", "1x0e+1x1o+1x2e", "4x1o+8x2e+8x1o", [(1, 1, 0), (0, 1, 1), (0, 2, 2), (0, 0, 2)]), 0),
    (("4x0e+4x1o", "1x0e+1x1o", "4x0e+4x1o", [(0, 0, 0)] * 65), 2),    # more than 64 paths
    (("4x0e+4x1o", "1x0e+1x1o", "4x0e+4x1o", [(1, 1, 0), (0, 0, 0)]), "uvw"),   # uvw, runtime path table
    (("4x0e+8x1o", "1x0e+1x1o", "4x0e+4x1o", [(1, 1, 0), (0, 0, 0)]), "uvw-2"),  # uvw: one mul per side
    (("4x0e+4x1o", "1x0e+1x1o", "4x0e+4x1o", [(0, 0, 2)]), 1),          # index out of range
])
def test_plan_validation(tp, args, status):
    mode = "uvu"
    if isinstance(status, str):
        mode, status = "uvw", int(status[4:] or 0)
    if status == 0:
        tp.Plan(*args, mode)
        return
    with pytest.raises(tp.TPError) as ei:
        tp.Plan(*args, mode)
    assert ei.value.status == status, str(ei.value)


def test_path_table_plan_sizes(tp):
    """Blocks of different multiplicities: widths and the per-edge weight count follow the
    blocks of each path (uvu: the path's input multiplicity)."""
    plan = tp.Plan("8x1o+4x0e", "1x0e+1x1o+1x2e", "4x1o+8x2e+8x1o", [(1, 1, 0), (0, 1, 1), (0, 2, 2), (0, 0, 2)])
    assert plan.in_dim == 8 * 3 + 4
    assert plan.out_dim == 4 * 3 + 8 * 5 + 8 * 3
    assert plan.n_edge_weights == 4 + 8 + 8 + 8


def test_path_coeff_rejects_nan(tp):
    spec = synth.CONFIGS["c1"]
    with pytest.raises(tp.TPError):
        tp.Plan(spec.irreps_in, spec.irreps_sh, spec.irreps_out, spec.paths, "uvu",
                path_coeff=[1.0, float("nan"), 1.0, 1.0])


def test_workspace_contract(tp):
    spec = synth.CONFIGS["c2"]
    plan = tp.Plan(spec.irreps_in, spec.irreps_sh, spec.irreps_out, spec.paths)
    N, E = 1536, 46080
    assert tp.tp_workspace_size(plan, N, E, tp.TP_OP_FWD) == 0
    for op in (tp.TP_OP_BWD, tp.TP_OP_DBWD):
        b = tp.tp_workspace_size(plan, N, E, op)
        # int32 graph indices only: perm, the radix sort's id buffer and its digit counts
        # (at most 4 bytes per edge plus one 2,048-entry row), colptr, alignment
        assert 8 * E <= b <= 12 * E + 4 * (N + 1) + 4 * 2 * 2048 + 6 * 256


def test_transpose_workspace_is_int_sized(tp):
    # one 11-bit pass up to 2,047 nodes (no second id buffer), then two passes
    assert tp.tp_csr_transpose_workspace_size(1536, 46080) == 4 * 2048 * (23 + 1)
    assert tp.tp_csr_transpose_workspace_size(100_000, 3_001_138) == 4 * (3_001_138 + 512 * (1466 + 1))
    assert tp.tp_csr_transpose_workspace_size(0, 0) == 4 * 2
    for N, E in ((24, 192), (4096, 162_892), (8192, 294_643), (2**31 - 1, 2**31 - 1)):
        assert tp.tp_csr_transpose_workspace_size(N, E) <= 8 * E + 4 * 2 * 2048
    with pytest.raises(tp.TPError):
        tp.tp_csr_transpose_workspace_size(-1, 4)


def test_uvw_multiplicities_off_the_tma_pitch_take_the_path_table(tp):
    # the compiled mixing GEMMs load rows by TMA, whose row pitch must be a multiple of 16
    # bytes; other multiplicities run through the path table (node-sized x W, no TMA)
    spec = synth.CONFIGS["c4"]
    odd_in = "+".join(f"30x{b.split('x')[1]}" for b in spec.irreps_in.split("+"))
    plan = tp.Plan(odd_in, spec.irreps_sh, spec.irreps_out, spec.paths, "uvw")
    assert plan.n_shared_weights == len(spec.paths) * 30 * 128
    N, E = 1000, 30000
    # forward workspace: x W per path (N x sum_p d1_p x mul_out floats), node sized
    assert tp.tp_workspace_size(plan, N, E, tp.TP_OP_FWD) <= 4 * N * 51 * 128 + 1024
    ok_in = "+".join(f"36x{b.split('x')[1]}" for b in spec.irreps_in.split("+"))
    tp.Plan(ok_in, spec.irreps_sh, spec.irreps_out, spec.paths, "uvw")


def test_uvw_workspace_is_node_sized(tp):
    spec = synth.CONFIGS["c4"]
    plan = tp.Plan(spec.irreps_in, spec.irreps_sh, spec.irreps_out, spec.paths, "uvw")
    N, E = 100_000, 3_001_138
    a_bytes = 4 * N * 51 * 128                   # per-path node state A (and its gradient G)
    f = tp.tp_workspace_size(plan, N, E, tp.TP_OP_FWD)
    b = tp.tp_workspace_size(plan, N, E, tp.TP_OP_BWD)
    # fwd: A and W regrouped for the GEMM (TF32 hi and lo)
    assert a_bytes <= f <= a_bytes + 2 * 4 * plan.n_shared_weights + 4096
    # bwd: transpose ints (at most 12 bytes/edge + O(N)), A, G, x as K-contiguous rows, W
    # regrouped twice (hi and lo each), at most 64 split-K partials of gW
    x_bytes = 4 * N * plan.in_dim
    assert b <= 12 * E + 12 * (N + 1) + 2 * a_bytes + x_bytes + 68 * 4 * plan.n_shared_weights + 16 * 2048
    with pytest.raises(tp.TPError):
        tp.tp_workspace_size(plan, N, E, tp.TP_OP_DBWD)


def test_calls_reject_bad_arguments_before_the_device(lib, tp):
    spec = synth.CONFIGS["c1"]
    plan = tp.Plan(spec.irreps_in, spec.irreps_sh, spec.irreps_out, spec.paths)
    h = plan.handle
    fake = C.c_void_p(0x10000)     # never dereferenced: every call below fails host checks
    odd = C.c_void_p(0x10002)
    # null plan
    assert lib.tp_conv_fwd(None, 4, 8, fake, fake, fake, fake, fake, None, fake, None, 0, None) == 1
    # negative sizes
    assert lib.tp_conv_fwd(h, -1, 8, fake, fake, fake, fake, fake, None, fake, None, 0, None) == 1
    # null output
    assert lib.tp_conv_fwd(h, 4, 8, fake, fake, fake, fake, fake, None, None, None, 0, None) == 1
    # null edge inputs with E > 0
    assert lib.tp_conv_fwd(h, 4, 8, fake, None, fake, fake, fake, None, fake, None, 0, None) == 1
    # misaligned pointer
    assert lib.tp_conv_fwd(h, 4, 8, fake, fake, odd, fake, fake, None, fake, None, 0, None) == 1
    # N = 0 is a no-op
    assert lib.tp_conv_fwd(h, 0, 0, None, None, None, None, None, None, None, None, 0, None) == 0
    # backward: workspace too small
    st = lib.tp_conv_bwd(h, 4, 8, fake, fake, None, None, fake, fake, fake, None, fake, fake, fake, None, None,
                         fake, 16, None)
    assert st == 4
    # colptr without perm
    st = lib.tp_conv_bwd(h, 4, 8, fake, fake, fake, None, fake, fake, fake, None, fake, fake, fake, None, None,
                         fake, 1 << 20, None)
    assert st == 1
    # transpose: null outputs
    assert lib.tp_csr_transpose(4, 8, None, fake, None, fake, fake, 1 << 20, None) == 1
    msg = lib.tp_last_error_message()
    assert msg and b"null" in msg.lower()
    # over int32 range
    assert lib.tp_conv_fwd(h, 1 << 31, 8, fake, fake, fake, fake, fake, None, fake, None, 0, None) == 2


def test_no_cpu_fallback_without_device(lib, tp):
    """A call that passes host checks goes to CUDA; with no device it fails loudly."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("device present")
    spec = synth.CONFIGS["c1"]
    plan = tp.Plan(spec.irreps_in, spec.irreps_sh, spec.irreps_out, spec.paths, flags=tp.TP_FLAG_CHECK_INDICES)
    fake = C.c_void_p(0x10000)
    st = lib.tp_conv_fwd(plan.handle, 4, 8, fake, fake, fake, fake, fake, None, fake, fake, 256, None)
    assert st == 5
    assert b"cuda" in lib.tp_last_error_message().lower() or lib.tp_last_error_message()


def test_device_error_word_without_a_plan(lib):
    """plan NULL reads the per-device word (used by the linear maps); code NULL is rejected
    first; without a device the read fails loudly instead of reporting 0."""
    import torch
    code = C.c_int32(-1)
    assert lib.tp_get_device_error(None, None, None, None) == 1
    if not torch.cuda.is_available():
        assert lib.tp_get_device_error(None, None, None, C.byref(code)) == 5


def test_bounded_wait_check_rejects_bad_arguments_before_the_device(lib):
    res = C.c_int32(-1)
    assert lib.tp_check_bounded_waits(0, None, C.byref(res)) == 1
    assert lib.tp_check_bounded_waits(2_000_000_000, None, C.byref(res)) == 1
    assert lib.tp_check_bounded_waits(1000, None, None) == 1


def test_missing_library_fails_loudly_on_first_call(tmp_path):
    """Without libtp.so the package still imports (so its build step can run), and the
    first call raises instead of computing anything another way."""
    import subprocess
    import sys
    code = (
        "import sys; sys.path.insert(0, %r)\n"
        "import equivariant_tensor_product_b200._lib as L\n"
        "L.LIB_PATH = %r\n"
        "import equivariant_tensor_product_b200 as tp, synth\n"
        "s = synth.CONFIGS['c1']\n"
        "try:\n"
        "    tp.Plan(s.irreps_in, s.irreps_sh, s.irreps_out, s.paths)\n"
        "except ImportError as e:\n"
        "    print('ImportError', e)\n"
    ) % (ROOT, str(tmp_path / "libtp.so"))
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300)
    assert "ImportError" in out.stdout and "libtp.so is missing" in out.stdout, (out.stdout, out.stderr)


def test_gaunt_plan_contract(tp):
    g = tp.Gaunt("32x0e+32x1o+32x2e", 2, "32x0e+32x1o+32x2e")
    assert (g.in_dim, g.out_dim, g.n_edge_weights, g.grid_points) == (288, 288, 96, 28)
    assert tp.Gaunt("4x1o", 1, "4x0e").grid_points == 8
    assert tp.Gaunt("4x3o", 0, "4x3o").grid_points == 50
    N, E = 1000, 30000
    f = tp.tp_gaunt_workspace_size(g, N, E, tp.TP_OP_FWD)
    b = tp.tp_gaunt_workspace_size(g, N, E, tp.TP_OP_BWD)
    assert 4 * N * 28 * 32 <= f <= 4 * N * 28 * 32 + 256            # node sized
    assert b <= 2 * f + 12 * E + 8 * (N + 1) + 4 * 2 * 2048 + 1024
    for args, status in ((("4x1e", 1, "4x0e"), 1), (("4x0e+8x1o", 1, "4x0e"), 1), (("4x0e", 1, "8x0e"), 1),
                         (("4x4e", 1, "4x0e"), 2), (("4x0e", 4, "4x0e"), 2), (("256x0e", 1, "256x0e"), 2),
                         (("4x1o+4x0e", 1, "4x0e"), 1)):
        with pytest.raises(tp.TPError) as e:
            tp.Gaunt(*args)
        assert e.value.status == status, args


def test_radial_contract_on_the_host(lib, tp):
    """The fused radial projection: hidden widths, plan modes and arguments are checked before
    the device; the backward workspace is the transpose region plus W_r-sized regions (W_r
    transposed and at most 256 gW_r partials), nothing edge x feature sized."""
    spec = synth.CONFIGS["c2"]
    plan = tp.Plan(spec.irreps_in, spec.irreps_sh, spec.irreps_out, spec.paths)
    N, E, H, nw = 1536, 46080, 64, plan.n_edge_weights
    assert tp.tp_radial_workspace_size(plan, N, E, H, tp.TP_OP_FWD) == 0
    b = tp.tp_radial_workspace_size(plan, N, E, H, tp.TP_OP_BWD)
    base = tp.tp_workspace_size(plan, N, E, tp.TP_OP_BWD)
    extra = b - base
    assert 4 * H * nw * 2 <= extra <= 4 * H * nw * 257 + 512
    assert tp.tp_radial_workspace_size(plan, 10 * N, 10 * E, H, tp.TP_OP_BWD) - tp.tp_workspace_size(
        plan, 10 * N, 10 * E, tp.TP_OP_BWD) <= 4 * H * nw * 257 + 512
    for bad_h in (0, 3, 68):
        with pytest.raises(tp.TPError):
            tp.tp_radial_workspace_size(plan, N, E, bad_h, tp.TP_OP_FWD)
    with pytest.raises(tp.TPError):
        tp.tp_radial_workspace_size(plan, N, E, H, tp.TP_OP_DBWD)
    c4 = synth.CONFIGS["c4"]
    uvw = tp.Plan(c4.irreps_in, c4.irreps_sh, c4.irreps_out, c4.paths, "uvw")
    with pytest.raises(tp.TPError):
        tp.tp_radial_workspace_size(uvw, N, E, H, tp.TP_OP_FWD)
    h = plan.handle
    fake, odd, off8 = C.c_void_p(0x10000), C.c_void_p(0x10002), C.c_void_p(0x10008)
    # hidden width not a multiple of 4: unsupported
    assert lib.tp_conv_fwd_radial(h, 4, 8, 6, fake, fake, fake, fake, fake, fake, fake, None, 0, None) == 2
    # null output, null edge inputs with E > 0, misaligned pointers, h not on 16 bytes
    assert lib.tp_conv_fwd_radial(h, 4, 8, 8, fake, fake, fake, fake, fake, fake, None, None, 0, None) == 1
    assert lib.tp_conv_fwd_radial(h, 4, 8, 8, fake, None, fake, fake, fake, fake, fake, None, 0, None) == 1
    assert lib.tp_conv_fwd_radial(h, 4, 8, 8, fake, fake, odd, fake, fake, fake, fake, None, 0, None) == 1
    assert lib.tp_conv_fwd_radial(h, 4, 8, 8, fake, fake, fake, fake, off8, fake, fake, None, 0, None) == 1
    # N = 0 is a no-op
    assert lib.tp_conv_fwd_radial(h, 0, 0, 8, None, None, None, None, None, None, None, None, 0, None) == 0
    # backward: workspace too small
    st = lib.tp_conv_bwd_radial(h, 4, 8, 8, fake, fake, None, None, fake, fake, fake, fake, fake, fake, fake,
                                fake, None, fake, 16, None)
    assert st == 4
