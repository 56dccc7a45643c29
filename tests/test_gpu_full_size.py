"""Parity at the workloads' full sizes, every row.

The prefill (T=8192, H=2048, I=768, E=128, k=8) and wide (T=4096, H=2048,
I=512, E=512, k=10) forwards are checked on every row of G, U, h and y and
every token of out, on each tile path: these sizes reach the full tile
counts, the persistent schedules' tails and the split-K choices that the
reduced shapes of the every-row tests do not.  The skewed workload (T=16384,
H=4096, I=1408, E=64, k=6) is checked on every row of its hottest expert, a
median one and its smallest non-empty one, in the forward and the backward
chain, with every token that selects the median or the smallest expert and
the first 64 tokens of the hottest (every token holds a row of the hottest
expert, and the oracle's full skewed forward takes minutes on the host).

Each step is compared with the oracle on the device's own inputs of that
step, and the end-to-end output with the oracle's chain (tests/helpers.py:
2e-2 * rms, beyond it only justified rounding flips).
"""
import numpy as np
import pytest

import oracle
from helpers import check_forward_steps, check_routing, generated, gpu_forward_numpy, values_in
from moe_routed_experts_b200 import binding as B

pytestmark = pytest.mark.gpu

_ORACLE = {}


def _oracle_full(name):
    """The oracle's full forward of one workload, computed once and shared by
    the three paths (about 1.3 GB of host arrays for prefill and wide)."""
    if name not in _ORACLE:
        _ORACLE[name] = oracle.forward(generated(name))
    return _ORACLE[name]


@pytest.fixture(params=[1, 2, 3], ids=["warp_tiles", "tcgen05_tiles", "tcgen05_pair_tiles"])
def path(request):
    try:
        prev = B.set_projection_path(request.param)
    except ValueError:
        pytest.skip("projection path %d not available" % request.param)
    yield request.param
    B.set_projection_path(prev)


@pytest.mark.parametrize("name", ["prefill", "wide"])
def test_forward_every_row_full_size(name, path):
    inp = generated(name)
    res, _, _ = gpu_forward_numpy(inp)
    want = _oracle_full(name)
    check_routing(res, want, name)
    assert np.array_equal(res["values"], values_in(res["values_dt"], want["values"]))
    check_forward_steps(inp, res, want, "%s/path%d" % (name, path))
    assert res["status"] == 0


def skewed_rows_and_tokens(offsets, row_of, selected, expert_start=0, hot_tokens=64):
    """Rows of the hottest, a median and the smallest non-empty expert, and
    the tokens that select the latter two plus the first `hot_tokens` that
    select the hottest."""
    counts = np.diff(offsets)
    nz = np.nonzero(counts)[0]
    by_count = nz[np.argsort(counts[nz], kind="stable")]
    hot, small, median = int(by_count[-1]), int(by_count[0]), int(by_count[len(by_count) // 2])
    rows = np.concatenate([np.arange(offsets[e], offsets[e + 1]) for e in sorted({hot, median, small})])
    local = selected.astype(np.int64) - expert_start
    hit = lambda e: np.nonzero(np.any(local == e, axis=1))[0]
    tokens = np.union1d(np.union1d(hit(median), hit(small)), hit(hot)[:hot_tokens])
    return rows.astype(np.int64), tokens.astype(np.int64), (hot, median, small)


def test_forward_skewed_hot_median_smallest_experts_every_row(path):
    inp = generated("skewed")
    w = inp["workload"]
    res, _, _ = gpu_forward_numpy(inp)
    rows, tokens, experts = skewed_rows_and_tokens(res["offsets"], res["row_of"], res["selected"], w.expert_start)
    want = oracle.forward(inp, rows=rows, tokens=tokens)
    check_routing(res, want, "skewed")
    check_forward_steps(inp, res, want, "skewed/path%d experts %s" % (path, experts), rows=want["rows_used"],
                        tokens=tokens)
    assert res["status"] == 0
