"""Checks against values the KVSlimmer pages print (fixtures under tests/golden/)."""

import os

from asymmetric_kv_merging_b200 import accounting
from asymmetric_kv_merging_b200.inputs import WORKLOADS

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
UNIT = {"bytes": 1, "KiB": 1 << 10, "GiB": 1 << 30}


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [line.split() for line in f if line.strip() and not line.startswith("#")]


def test_kv_cache_memory_table():
    for layers, heads, dim, eb, batch, tokens, value, unit in _rows("kv_cache_memory.txt"):
        got = accounting.kv_cache_bytes(layers, heads, dim, eb, tokens, batch)
        # the page rounds to whole KiB / GiB ("约", "~")
        assert round(got / UNIT[unit]) == int(value), (tokens, got)


def test_workloads_protect_the_pages_sink_tokens():
    settings = {k: int(v) for k, v in _rows("experiment_settings.txt")}
    for w in WORKLOADS:
        assert w.sink == settings["preserved_initial_tokens"]


def test_prefill_measurement_uses_the_pages_compression_setting():
    """bench.py --prefill runs the setting the pages' experiments use: budget 2048,
    chunk 512, 32 preserved initial tokens."""
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    if root not in sys.path:
        sys.path.insert(0, root)
    import bench
    settings = {k: int(v) for k, v in _rows("experiment_settings.txt")}
    assert bench.PREFILL["budget"] == settings["default_budget_tokens"]
    assert bench.PREFILL["chunk"] == settings["default_chunk_tokens"]
    assert bench.PREFILL["sink"] == settings["preserved_initial_tokens"]
