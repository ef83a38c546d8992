"""The GPU parity gates, exercised on the CPU: the checks in svdq_cases that every
`-m gpu` test relies on must pass the oracle's own results and reject each kind of
wrong result a kernel could produce -- one flipped code, a changed block scale, a
`t` or `y` element two bf16 ulps off, a non-finite output, many small errors that
stay under the elementwise bound but break rel-L2 -- and the sampled rows must
cover every 128-row M tile.  The "GPU" results here are the oracle's, perturbed."""
import numpy as np
import pytest

import oracle
import workloads as wl
from svdq_cases import (assert_t_close, assert_y_close, bf, bf16_ulp, check_layer_output, int4_bytes_to_packed,
                        oracle_layer, tile_rows)


class _FakeDeviceLayer:
    """Stands in for GpuLayer: read_act returns given (possibly perturbed) results."""

    def __init__(self, act):
        self.act = act

    def read_act(self, M):
        return dict(codes=self.act["codes"].copy(), scales=self.act["scales"].copy(), t=self.act["t"].copy(),
                    g_x=self.act["g_x"])


def _case(fmt):
    X, W, b, prep = oracle_layer(wl.small_layer(300, 512, 192, 32, fmt, layer_id=71))
    act = oracle.quantize_act(X, prep)
    y = oracle.forward_from_act(act, prep)
    return X, prep, act, y


def _bump(bits, ulps):
    """bf16 bit patterns moved `ulps` units away from zero (same sign, finite here)."""
    return (bits.astype(np.int32) + ulps).astype(np.uint16)


@pytest.mark.parametrize("fmt", ["int4", "nvfp4"])
def test_oracle_results_pass(fmt):
    X, prep, act, y = _case(fmt)
    s = check_layer_output(_FakeDeviceLayer(act), X, prep, y, tile_rows(X.shape[0], 0))
    assert s["n_flip"] == 0 and s["rel_l2"] == 0.0


@pytest.mark.parametrize("fmt", ["int4", "nvfp4"])
def test_a_flipped_code_is_rejected(fmt):
    X, prep, act, y = _case(fmt)
    bad = dict(act, codes=act["codes"].copy())
    bad["codes"][123, 45] ^= 0x01
    with pytest.raises(AssertionError):
        check_layer_output(_FakeDeviceLayer(bad), X, prep, y)


@pytest.mark.parametrize("fmt", ["int4", "nvfp4"])
def test_a_changed_scale_is_rejected(fmt):
    X, prep, act, y = _case(fmt)
    bad = dict(act, scales=act["scales"].copy())
    bad["scales"][7, 1] += 1
    with pytest.raises(AssertionError):
        check_layer_output(_FakeDeviceLayer(bad), X, prep, y)


def test_t_two_ulps_off_beyond_its_bound_is_rejected():
    X, prep, act, y = _case("nvfp4")
    t = act["t"].copy()
    t[5, 3] = _bump(t[5:6, 3], 2)[0]
    # the summation allowance of that element is far below two bf16 ulps here
    with pytest.raises(AssertionError):
        assert_t_close(t, act["t"])
    assert_t_close(_bump(act["t"], 1), act["t"])  # one ulp (the final rounding) is allowed


def test_y_element_past_the_gate_is_rejected():
    X, prep, act, y = _case("nvfp4")
    o = bf(y)
    i, j = np.unravel_index(np.argmax(np.abs(o)), o.shape)
    lim = 2e-2 + bf16_ulp(o[i, j])
    step = bf16_ulp(o[i, j])
    k = int(np.ceil(lim / step)) + 1  # enough ulps to pass 2e-2 + 1 ulp
    bad = y.copy()
    bad[i, j] = _bump(y[i:i + 1, j], k)[0]
    with pytest.raises(AssertionError):
        assert_y_close(bad, y)
    ok = y.copy()
    ok[i, j] = _bump(y[i:i + 1, j], 1)[0]
    assert_y_close(ok, y)  # one ulp anywhere is within the gate


def test_many_small_errors_break_rel_l2():
    X, prep, act, y = _case("nvfp4")
    o = bf(y)
    noisy = o + np.where(np.abs(o) > 0, 0.9 * 2e-2, 0.0) * np.sign(np.random.default_rng(0).standard_normal(o.shape))
    bad = oracle.f64_to_bf16(noisy)
    assert np.all(np.abs(bf(bad) - o) <= 2e-2 + bf16_ulp(o))  # every element inside the elementwise bound
    with pytest.raises(AssertionError):
        assert_y_close(bad, y)


def test_non_finite_output_is_rejected():
    X, prep, act, y = _case("int4")
    bad = y.copy()
    bad[0, 0] = 0x7FC0
    with pytest.raises(AssertionError):
        assert_y_close(bad, y)


@pytest.mark.parametrize("M", [1, 127, 128, 129, 300, 4608, 9216 + 17])
def test_sampled_rows_cover_every_tile(M):
    rows = tile_rows(M, 3)
    assert rows.min() >= 0 and rows.max() < M
    assert set(range((M + 127) // 128)) <= set((rows // 128).tolist())
    assert 0 in rows and M - 1 in rows


def test_int4_device_bytes_must_be_canonical():
    good = np.array([[0x00, 0x38, 0xB8, 0x40, 0xD0, 0x4E]], np.uint8)  # 0, 1, -1, 2, -8, 7 as E4M3
    np.testing.assert_array_equal(int4_bytes_to_packed(good), [[0x10, 0x2F, 0x78]])
    for bad in (0x80, 0x3C, 0x50):  # negative zero, 1.5, 8 (out of range)
        with pytest.raises(AssertionError):
            int4_bytes_to_packed(np.array([[bad, 0x00]], np.uint8))
