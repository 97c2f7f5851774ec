"""Host-side logic of the benchmark and the step driver, on the CPU: layer
grouping of the end-to-end step, the expected verified tokens per step
against the planted-acceptance sampler, and the clock record's parsing."""
import numpy as np
import pytest

import bench
from lossless_diffusion_speculative_b200 import workloads as wl
from lossless_diffusion_speculative_b200.step import layer_groups


@pytest.mark.parametrize("L,chunk", [(36, (1, 8, 9)), (36, 9), (5, (2,)), (3, (1, 2)), (7, (10,)), (4, 1)])
def test_layer_groups_cover_every_layer_once_in_order(L, chunk):
    groups = layer_groups(L, chunk)
    assert [l for g in groups for l in g] == list(range(L))
    sizes = [len(g) for g in groups]
    want = [chunk] if isinstance(chunk, int) else list(chunk)
    for k, n in enumerate(sizes[:-1]):                       # all but the last group are full
        assert n == want[min(k, len(want) - 1)]
    assert 1 <= sizes[-1] <= want[min(len(sizes) - 1, len(want) - 1)]


@pytest.mark.parametrize("plant", ["uniform", "geom:0.14285714285714285", "geom:0.1111111111111111",
                                   "half", "fixed:3", "fixed:40"])
def test_expected_tokens_match_the_planted_sampler(plant):
    """The closed forms of E[sum_b min(a_b + 1, K)] agree with the mean of the
    seeded sampler over many sequences (within 5 standard errors)."""
    w = wl.WORKLOADS["qwen3_8b_step"].with_(B=40000, plant=plant)
    a = wl.planted_accept_lengths(w)
    per = np.minimum(a + 1, w.K).astype(np.float64)
    exp = wl.expected_tokens_per_step(w) / w.B
    se = per.std() / np.sqrt(w.B)
    assert abs(per.mean() - exp) <= 5 * se + 1e-12, (per.mean(), exp, se)


def test_expected_tokens_of_the_headline_step():
    """Uniform a in {0..32}, K = 32: (sum_{a<32} (a + 1) + 32) / 33 = 560 / 33."""
    w = wl.WORKLOADS["qwen3_8b_step"]
    assert wl.expected_tokens_per_step(w) == pytest.approx(560 / 33)


class _Done:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0


def test_clock_record_uses_busy_samples_and_collects_reasons():
    cs = bench.ClockSampler("GPU-0")
    cs.proc = _Done()
    idle = "345, 1965, 150.0, 0x0, Not Active, Not Active, Not Active, Not Active, 0"
    busy = ["1965, 1965, 700.0, 0x0, Not Active, Not Active, Not Active, Not Active, 100",
            "1950, 1965, 900.0, 0x4, Not Active, Not Active, Not Active, Active, 99",
            "1965, 1965, 650.0, 0x0, Not Active, Not Active, Not Active, Not Active, 97"]
    cs.lines = [idle, idle] + busy + [idle, "garbage line", ""]
    rec = cs.stop()
    assert rec["samples"] == 6 and rec["samples_under_load"] == 3
    assert rec["sm_mhz"] == 1965.0 and rec["sm_max_mhz"] == 1965.0
    assert rec["reasons"] == ["sw_power_cap"]
    assert rec["power_w_max"] == 900.0


def test_clock_record_without_samples_says_so():
    cs = bench.ClockSampler("GPU-0")
    rec = cs.stop()
    assert rec["samples"] == 0 and rec["sm_mhz"] is None
