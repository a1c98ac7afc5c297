"""Host logic of bench.py's CPU-oracle timing: the sample is sized for a target time."""
import os
import sys
import types

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _fake_run(sec_per_token, log):
    def run(n):
        log.append(n)
        return n * sec_per_token
    return run


def test_sample_grows_to_the_target_and_is_capped():
    log = []
    tok, secs, n = bench.sized_oracle_sample(_fake_run(0.01, log), 2048, 10.0)
    # 100 tokens/s: a 16-token probe, then 1000 tokens for about 10 s in one pass
    assert log == [16, 1000] and (tok, n) == (1000, 1000) and abs(secs - 10.0) < 1e-9


def test_short_workload_repeats_passes_until_the_target():
    log = []
    tok, secs, n = bench.sized_oracle_sample(_fake_run(0.001, log), 2048, 10.0)
    # 1000 tokens/s: capped at the 2048 prepared tokens, passes repeat until >= 0.8 * target
    assert n == 2048 and log[0] == 16 and all(m == 2048 for m in log[1:])
    assert secs >= 8.0 and tok == 2048 * (len(log) - 1) and abs(tok / secs - 1000.0) < 1e-6


def test_fewer_tokens_than_the_probe():
    log = []
    tok, secs, n = bench.sized_oracle_sample(_fake_run(1.0, log), 5, 10.0)
    assert log[0] == 5 and n == 5 and tok % 5 == 0


def test_reference_steps_fit_in_two_minutes():
    for steps, want in [(1, 10.0), (12, 10.0), (20, 6.0), (1000, 0.5)]:
        args = types.SimpleNamespace(cpu_seconds=10.0, steps=steps)
        assert bench.reference_step_seconds(args) == want
