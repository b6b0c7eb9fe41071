"""bench.py's reference arm on CPU: the oracle timed on a bounded sample of
the workload prints one JSON line with the contract's keys (impl, the
cpu_baseline it describes, an e2e of its own value with no copies), and the
sampler covers the modulation-projection workloads."""

import importlib.util
import json
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("config", ["tiny_adarms", "style_stack18"])
def test_reference_line(config, capsys, monkeypatch):
    monkeypatch.setenv("RANK", "0")
    b = _bench()

    class Args:
        steps, warmup, gpus = 3, 3, 1

    Args.config = config
    assert b.run_reference(Args()) == 0
    lines = [l for l in capsys.readouterr().out.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["steps"] == 3 and d["warmup"] == 3
    assert d["value"] > 0 and d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["cores"] >= 1 and d["cpu_baseline"]["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    assert d["config"]["workload"].startswith(config)
    if config.startswith("style"):
        assert d["dtype"].startswith("bf16")


def test_style_sampler_is_bounded():
    """The projection's sample is a leading block of output columns; its
    tokens count the share of the columns it covers."""
    from fp8_transformer_block_b200 import synth
    b = _bench()
    w = synth.WORKLOADS["style_vla18"]
    fn, tokens, text = b.oracle_sampler("style_stack18", synth, rows_cap=1536)
    fn()
    ws = synth.WORKLOADS["style_stack18"]
    assert tokens == pytest.approx(ws.rows * 1536 / ws.N)
    assert text.startswith("1536 of 56832")
    assert w.N == 37 * 3 * 2048
