"""The float64 oracle, pinned to facts that do not come from itself (CPU only).

Every pin in ``_pins.py`` runs on both write-ups of the oracle (C and NumPy);
the two are also compared with each other; and copies of the C oracle with a
planted mistake (wrong sign, dropped term, transposed operand, wrong index
map ...) are compiled on the fly to show that each such mistake fails at
least one pin.
"""
import math
import os

import numpy as np
import pytest

import oracle
from oracle import ss2d_oracle_np as onp
import _pins
from selective_scan_ss2d_b200 import workloads as wl

IMPLS = {
    "c": (oracle.ss2d_forward, oracle.selective_scan_fwd),
    "numpy": (onp.ss2d_forward, onp.selective_scan_fwd),
}


@pytest.mark.parametrize("pin", _pins.ALL_PINS, ids=lambda f: f.__name__)
@pytest.mark.parametrize("impl", sorted(IMPLS))
def test_pin(impl, pin):
    pin(IMPLS[impl])


def test_scan_orders_fixture():
    g = _pins.read_golden("scan_orders_2x3.txt")
    H, W = 2, 3
    np_orders = onp.scan_orders_2d(H, W)
    arr_orders = _pins.array_scan_orders(H, W)
    for k in range(4):
        want = [int(v) for v in g[f"k{k}"]]
        got_c = [oracle.scan_pixel(0, k, l, H, W) for l in range(H * W)]
        assert got_c == want
        assert list(np_orders[k]) == want
        assert list(arr_orders[k]) == want


@pytest.mark.parametrize("H,W", [(1, 1), (1, 6), (5, 1), (3, 7), (8, 8), (6, 4)])
def test_scan_orders_are_permutations_and_agree(H, W):
    np_orders = onp.scan_orders_2d(H, W)
    for k in range(4):
        got = np.array([oracle.scan_pixel(0, k, l, H, W) for l in range(H * W)])
        assert sorted(got) == list(range(H * W))
        assert np.array_equal(got, np_orders[k])
    L = H * W
    for k in range(2):
        got = [oracle.scan_pixel(1, k, l, 1, L) for l in range(L)]
        assert got == list(onp.scan_orders_1d(L)[k])


@pytest.mark.parametrize("K,N", [(1, 6), (2, 6), (4, 6), (4, 40)])
def test_c_and_numpy_writeups_agree_2d(K, N):
    rng = np.random.default_rng(100 + K + N)
    p = _pins.rand_problem(rng, 2, 3, 5, 3, K, N)
    yc, dc = _pins.call2d(IMPLS["c"], p, K=K, return_dirs=True)
    yn, dn = _pins.call2d(IMPLS["numpy"], p, K=K, return_dirs=True)
    np.testing.assert_allclose(yc, yn, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dc, dn, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("K,N", [(1, 16), (2, 16), (2, 64)])
def test_c_and_numpy_writeups_agree_1d(K, N):
    rng = np.random.default_rng(200 + K + N)
    p = _pins.rand_problem(rng, 2, 3, 1, 37, K, N, one_d=True)
    yc = _pins.call1d(IMPLS["c"], p, K=K)
    yn = _pins.call1d(IMPLS["numpy"], p, K=K)
    np.testing.assert_allclose(yc, yn, rtol=1e-12, atol=1e-12)


def test_threads_do_not_change_the_result():
    rng = np.random.default_rng(7)
    p = _pins.rand_problem(rng, 3, 5, 4, 6, 4, 8)
    y1 = _pins.call2d(IMPLS["c"], p, K=4, threads=1)
    y4 = _pins.call2d(IMPLS["c"], p, K=4, threads=4)
    assert np.array_equal(y1, y4)


def test_oracle_rejects_bad_arguments():
    lib = oracle.lib()
    z = np.zeros(16)
    ptr = oracle._ptr(z)
    assert lib.oracle_ss2d_forward(*([ptr] * 7), ptr, None, 1, 1, 2, 2, 1, 3, 0, 1) == -4
    assert lib.oracle_selective_scan_fwd(*([ptr] * 7), ptr, None, 1, 1, 4, 1, 4, 0, 1) == -4
    assert lib.oracle_ss2d_forward(*([ptr] * 7), None, None, 1, 1, 2, 2, 1, 4, 0, 1) == -1
    assert lib.oracle_ss2d_forward(*([ptr] * 7), ptr, None, 1, 1, 2, 2, 0, 4, 0, 1) == -2


# ---------------------------------------------------------------------------
# planted mistakes: each edit of the C source must fail at least one pin
# ---------------------------------------------------------------------------
MUTATIONS = {
    "A_sign": ("const double A = -exp(A_log_row[n]);",
               "const double A = exp(A_log_row[n]);"),
    "A_not_exponentiated": ("const double A = -exp(A_log_row[n]);",
                            "const double A = -A_log_row[n];"),
    "dA_without_dt": ("const double dA = exp(dt * A);", "const double dA = exp(A);"),
    "dB_without_dt": ("dB = dt * Bv;\n", "dB = Bv;\n"),
    "input_dropped": ("h[n] = dA * h[n] + dB * u;", "h[n] = dA * h[n] + dB;"),
    "state_not_decayed": ("h[n] = dA * h[n] + dB * u;", "h[n] = h[n] + dB * u;"),
    "C_replaced_by_B": ("acc += C_dir[(int64_t)n * L + l] * h[n];",
                        "acc += B_dir[(int64_t)n * L + l] * h[n];"),
    "skip_dropped": ("y_pix[p] = acc + Dskip * u;", "y_pix[p] = acc;"),
    "bias_dropped": ("oracle_softplus(delta_seq[l] + dbias)",
                     "oracle_softplus(delta_seq[l])"),
    "softplus_is_exp": ("    return log1p(exp(z));", "    return exp(z);"),
    "column_map_transposed": ("return h * W + w;", "return w * H + h;"),
    "k3_not_reversed": ("    if (k == 3)\n        l = L - 1 - l;\n", ""),
    "k1_not_reversed": ("return (k % 2 == 0) ? l : (L - 1 - l);", "return l;"),
    "merge_overwrites": ("y_pix[p] += yk[p];", "y_pix[p] = yk[p];"),
    "B_time_index_shifted": ("const double Bv = B_dir[(int64_t)n * L + l];",
                             "const double Bv = B_dir[(int64_t)n * L + (l + 1) % L];"),
    "state_not_reset": ("    for (int n = 0; n < N; ++n)\n        h[n] = 0.0;\n", ""),
    "params_of_direction_0": ("const int64_t kd = (int64_t)k * D + d;",
                              "const int64_t kd = d;"),
    "gate_is_sigmoid": ("        return z / (1.0 + exp(-z));",
                        "        return 1.0 / (1.0 + exp(-z));"),
    "gate_sign_flipped": ("    return z * e / (1.0 + e);", "    return -z * e / (1.0 + e);"),
    "gate_skipped": ("        y[i] *= oracle_silu(z[i]);", "        y[i] *= 1.0;"),
}


@pytest.fixture(scope="module")
def variant_dir(tmp_path_factory):
    return tmp_path_factory.mktemp("oracle_variants")


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, variant_dir):
    old, new = MUTATIONS[name]
    src = oracle.source_text()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    lib = oracle.compile_variant(src.replace(old, new),
                                 os.path.join(str(variant_dir), f"lib_{name}.so"))

    def f2(*a, **kw):
        return oracle.ss2d_forward(*a, _lib=lib, **kw)

    def f1(*a, **kw):
        return oracle.selective_scan_fwd(*a, _lib=lib, **kw)

    caught = []
    for pin in _pins.ALL_PINS:
        try:
            pin((f2, f1))
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"planted mistake '{name}' passed every pin"


# ---------------------------------------------------------------------------
# the shared input generator
# ---------------------------------------------------------------------------
def test_bf16_rounding_fixture():
    rows = []
    with open(os.path.join(_pins.GOLDEN, "bf16_rne.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                a, b = line.split()[:2]
                rows.append((int(a, 16), int(b, 16)))
    f32 = np.array([r[0] for r in rows], dtype=np.uint32).view(np.float32)
    got = wl.f32_to_bf16_bits(f32)
    assert [int(v) for v in got] == [r[1] for r in rows]
    back = wl.bf16_bits_to_f32(got)
    assert np.array_equal(back.view(np.uint32) >> 16, got.astype(np.uint32))


def test_workload_recipe():
    inp = wl.make_inputs("tiny_fp32", seed=0)
    cfg = inp.cfg
    assert inp.x.shape == (1, 8, 8, 8) and inp.delta.shape == (1, 4, 8, 64)
    assert inp.Bs.shape == (1, 4, 4, 64) and inp.A_log.shape == (32, 4)
    np.testing.assert_allclose(np.exp(inp.A_log[0]), [1, 2, 3, 4], rtol=1e-6)
    dt = np.array([_pins.softplus_ref(float(v)) for v in inp.delta_bias])
    assert dt.min() >= 1e-3 * (1 - 1e-5) and dt.max() <= 1e-1 * (1 + 1e-5)
    assert np.all(inp.Dskip == 1.0)
    again = wl.make_inputs("tiny_fp32", seed=0)
    assert np.array_equal(inp.x, again.x) and np.array_equal(inp.Cs, again.Cs)
    other = wl.make_inputs("tiny_fp32", seed=1)
    assert not np.array_equal(inp.x, other.x)
    assert cfg.updates == 8192


def test_half_workloads_round_the_float32_draws():
    """bf16 and f16 workloads are the float32 draws rounded to nearest-even
    (same seed, same order), and as_f64 gives back exactly those values."""
    base = wl.make_inputs("tiny_fp32", seed=2)
    f16 = wl.make_inputs(base.cfg.with_(dtype=wl.F16), seed=2)
    bf = wl.make_inputs(base.cfg.with_(dtype=wl.BF16), seed=2)
    assert f16.x.dtype == np.float16 and bf.x.dtype == np.uint16
    for name in wl.Inputs.STREAMED:
        a = getattr(base, name)
        assert np.array_equal(getattr(f16, name), a.astype(np.float16))
        assert np.array_equal(f16.as_f64()[name], a.astype(np.float16).astype(np.float64))
        assert np.array_equal(bf.as_f64()[name],
                              wl.bf16_bits_to_f32(wl.f32_to_bf16_bits(a)).astype(np.float64))
        # both roundings stay within half a unit in the last place of their format
        assert np.all(np.abs(f16.as_f64()[name] - a) <= np.abs(a) * 2.0 ** -11 + 2.0 ** -25)
    assert f16.cfg.in_bytes_per_elem == 2 and base.cfg.in_bytes_per_elem == 4
    z = wl.make_gate(f16.cfg, seed=2)
    assert z.dtype == np.float16
    assert np.array_equal(wl.gate_as_f64(z, f16.cfg), z.astype(np.float64))


def test_config_table_matches_the_workloads():
    c = wl.CONFIGS
    assert (c["vmamba_t_stage1"].B, c["vmamba_t_stage1"].D, c["vmamba_t_stage1"].L) == (8, 192, 3136)
    assert (c["vmamba_b_stage3"].B, c["vmamba_b_stage3"].D, c["vmamba_b_stage3"].L) == (64, 1024, 196)
    assert (c["highres_256"].D, c["highres_256"].L) == (192, 65536)
    assert (c["vim_s_bidir"].B, c["vim_s_bidir"].D, c["vim_s_bidir"].L, c["vim_s_bidir"].K) == (128, 768, 197, 2)
    assert c["vmamba_t_stage1"].updates == 308281344
    # x + delta + Bs + Cs read once (bf16), y written once (fp32), params
    assert abs(c["vmamba_t_stage1"].algorithmic_bytes - 73.9e6) < 0.1e6


def test_channel_subproblem_matches_full_oracle():
    cfg = wl.CONFIGS["tiny_fp32"].with_(B=2, D=3, H=3, W=5)
    inp = wl.make_inputs(cfg, seed=3)
    f = inp.as_f64()
    y = oracle.ss2d_forward(f["x"], f["delta"], f["A_log"], f["Bs"], f["Cs"],
                            f["Dskip"], f["delta_bias"], K=4)
    for (b, d) in [(0, 0), (1, 2), (0, 1)]:
        s = wl.channel_subproblem(inp, b, d).as_f64()
        ys = oracle.ss2d_forward(s["x"], s["delta"], s["A_log"], s["Bs"], s["Cs"],
                                 s["Dskip"], s["delta_bias"], K=4)
        assert np.array_equal(ys[0, 0], y[b, d])


def test_softplus_definition():
    for z in [-30.0, -5.0, -1e-3, 0.0, 1e-3, 2.0, 15.0, 30.0]:
        assert math.isclose(oracle.softplus(z), math.log1p(math.exp(z)), rel_tol=1e-15)
        assert math.isclose(float(onp.softplus(z)), math.log1p(math.exp(z)), rel_tol=1e-15)
    assert oracle.softplus(1000.0) == 1000.0


def test_states_split_into_groups():
    """The states of a channel never interact: y with N = 40 states equals the
    sum of the outputs of states 0..15, 16..31 and 32..39 run alone, with the
    skip term counted once (pins the oracle where N is above 16)."""
    rng = np.random.default_rng(9)
    B, D, H, W, K, N = 1, 3, 4, 5, 4, 40
    L = H * W
    x = rng.standard_normal((B, D, H, W))
    delta = rng.standard_normal((B, K, D, L))
    A_log = rng.uniform(-1, 1, (K * D, N))
    Bs = rng.standard_normal((B, K, N, L))
    Cs = rng.standard_normal((B, K, N, L))
    Dskip = rng.standard_normal(K * D)
    bias = rng.uniform(-1, 1, K * D)
    y = oracle.ss2d_forward(x, delta, A_log, Bs, Cs, Dskip, bias, K=4)
    parts = []
    for lo, hi in [(0, 16), (16, 32), (32, 40)]:
        parts.append(oracle.ss2d_forward(x, delta, A_log[:, lo:hi], Bs[:, :, lo:hi],
                                         Cs[:, :, lo:hi], np.zeros(K * D), bias, K=4))
    skip = oracle.ss2d_forward(x, delta, A_log[:, :1], Bs[:, :, :1], 0 * Cs[:, :, :1], Dskip,
                               bias, K=4)
    np.testing.assert_allclose(y, parts[0] + parts[1] + parts[2] + skip, rtol=1e-12, atol=1e-12)
