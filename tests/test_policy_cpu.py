"""Host logic of the measured policy map, without a GPU: installing, validating and
looking up tables through the C ABI, the dispatcher's argument checks, and the tuner's
M-list parsing, candidate set and range merging."""
import pytest

import weight_only_quantized_gemv_b200 as ql
from weight_only_quantized_gemv_b200 import tune

M_MAX = 2 ** 31 - 1


@pytest.fixture(autouse=True)
def _empty_table():
    ql.qlinear_policy_set([])
    yield
    ql.qlinear_policy_set([])


def _e(**kw):
    d = dict(fmt=4, N=4096, K=4096, m_lo=1, m_hi=16, strategy=0, warps_per_unit=0, ctas=0)
    d.update(kw)
    return d


def test_builtin_rule_without_table():
    assert ql.qlinear_policy_size() == 0
    d, from_table = ql.qlinear_policy_lookup(4, 1, 4096, 4096)
    assert not from_table and d["strategy"] == ql.QL_STRATEGY_GEMV
    assert (d["m_lo"], d["m_hi"]) == (1, 64)
    d, _ = ql.qlinear_policy_lookup(16, 64, 8192, 28672)
    assert d["strategy"] == ql.QL_STRATEGY_GEMV
    d, _ = ql.qlinear_policy_lookup(16, 65, 8192, 28672)
    assert d["strategy"] == ql.QL_STRATEGY_PREFILL and (d["m_lo"], d["m_hi"]) == (65, M_MAX)


def test_table_lookup_first_match_and_exact_shape():
    ql.qlinear_policy_set([
        _e(m_lo=1, m_hi=1, ctas=296),
        _e(m_lo=2, m_hi=8, warps_per_unit=2),
        _e(m_lo=1, m_hi=8, ctas=7),                       # shadowed by the two above
        _e(m_lo=9, m_hi=M_MAX, strategy=1),
        _e(fmt=2, m_lo=1, m_hi=M_MAX, strategy=1),
    ])
    assert ql.qlinear_policy_size() == 5
    d, t = ql.qlinear_policy_lookup(4, 1, 4096, 4096)
    assert t and d["ctas"] == 296 and d["m_hi"] == 1
    d, t = ql.qlinear_policy_lookup(4, 5, 4096, 4096)
    assert t and d["warps_per_unit"] == 2 and d["ctas"] == 0
    d, t = ql.qlinear_policy_lookup(4, 9, 4096, 4096)
    assert t and d["strategy"] == 1
    d, t = ql.qlinear_policy_lookup(2, 1, 4096, 4096)
    assert t and d["strategy"] == 1
    # other shapes and formats fall back to the rule
    assert not ql.qlinear_policy_lookup(4, 5, 4096, 4224)[1]
    assert not ql.qlinear_policy_lookup(8, 5, 4096, 4096)[1]
    assert not ql.qlinear_policy_lookup(4, 5, 4224, 4096)[1]


@pytest.mark.parametrize("bad,status", [
    (dict(fmt=3), 4), (dict(strategy=2), 4), (dict(m_lo=0), 2), (dict(m_lo=5, m_hi=4), 2),
    (dict(N=24), 2), (dict(K=100), 2), (dict(N=0), 2), (dict(warps_per_unit=3), 2),
    (dict(ctas=-1), 2),
])
def test_invalid_entries_are_rejected_whole(bad, status):
    ql.qlinear_policy_set([_e(ctas=11)])
    with pytest.raises(ql.QLinearError) as ei:
        ql.qlinear_policy_set([_e(m_lo=1, m_hi=1), _e(**bad)])
    assert ei.value.status == status
    assert ql.qlinear_policy_size() == 1                  # the old table stays
    assert ql.qlinear_policy_lookup(4, 3, 4096, 4096)[0]["ctas"] == 11


def test_c_abi_argument_checks():
    lib = ql._lib
    assert lib.qlinear_policy_set(None, 2) == 1
    assert lib.qlinear_policy_set(None, -1) == 2
    assert lib.qlinear_policy_set(None, 0) == 0
    e = ql.ql_policy_entry()
    assert lib.qlinear_policy_lookup(4, 1, 128, 128, None, None) == 1
    assert lib.qlinear_policy_lookup(5, 1, 128, 128, e, None) == 4
    assert lib.qlinear_policy_lookup(4, 0, 128, 128, e, None) == 2
    assert lib.qlinear_policy_lookup(4, 1, 128, 128, e, None) == 0
    a = 1 << 20
    mm = lib.qlinear_matmul
    assert mm(5, a, a, a, a, a, 1, 128, 128, a, 1 << 20, None, None) == 4
    assert mm(4, a, a, a, a, a, 0, 128, 128, a, 1 << 20, None, None) == 2
    # GEMV slices (rule, no fp16 buffer): the first slice's checks run before any device work
    assert mm(4, None, a, a, a, a, 100, 128, 128, a, 1 << 20, None, None) == 1
    assert mm(4, a, a, a, a, a, 100, 120, 128, a, 1 << 20, None, None) == 2
    # prefill by the rule (M > 64) with a buffer: the prefill checks run first
    assert mm(4, a, a, a, a, a, 100, 128, 128, a, 1 << 20, a + 8, None) == 3


# ---------------------------------------------------------------------------
# tuner host logic


def test_parse_lists():
    assert tune.parse_m_list("1-4,8, 16,8") == [1, 2, 3, 4, 8, 16]
    with pytest.raises(ValueError):
        tune.parse_m_list("0-2")
    assert tune.parse_shapes("4096x4096,8192X28672") == [(4096, 4096), (8192, 28672)]


def test_candidates():
    c = tune.candidates(4, 4, 148)
    assert c[0] == (0, 0, 0) and c[-1] == (1, 0, 0)
    assert (0, 0, 148) in c and (0, 0, 444) in c and (0, 2, 0) in c and (0, 4, 0) in c
    assert (0, 2, 0) not in tune.candidates(4, 1, 148)
    assert (0, 2, 0) not in tune.candidates(2, 4, 148)
    assert tune.candidates(8, 32, 148) == [(0, 0, 0), (1, 0, 0)]


def test_build_entries_merges_ranges():
    best = {1: (0, 0, 296), 2: (0, 2, 0), 3: (0, 2, 0), 4: (0, 2, 0), 16: (0, 0, 0),
            32: (0, 0, 0), 64: (1, 0, 0), 128: (1, 0, 0)}
    e = tune.build_entries(4, 512, 1024, best)
    spans = [(x["m_lo"], x["m_hi"], x["strategy"], x["warps_per_unit"], x["ctas"]) for x in e]
    assert spans == [(1, 1, 0, 0, 296), (2, 4, 0, 2, 0), (5, 32, 0, 0, 0), (33, M_MAX, 1, 0, 0)]
    # every M is covered exactly once and the table installs
    ql.qlinear_policy_set(e)
    for m in (1, 2, 4, 5, 16, 17, 32, 33, 64, 100, 10 ** 6):
        d, t = ql.qlinear_policy_lookup(4, m, 512, 1024)
        assert t
        assert sum(1 for x in e if x["m_lo"] <= m <= x["m_hi"]) == 1


def test_pick_keeps_the_rule_unless_beaten_by_the_margin():
    rule = (100.0, (0, 0, 0))
    assert tune.pick([rule, (99.0, (0, 2, 0)), (150.0, (1, 0, 0))], 0.02) == rule
    assert tune.pick([rule, (97.0, (0, 2, 0))], 0.02) == (97.0, (0, 2, 0))
    # the prefill strategy is taken whenever it is fastest (no margin)
    assert tune.pick([rule, (99.5, (1, 0, 0))], 0.02) == (99.5, (1, 0, 0))


def test_rule_choice_matches_the_library_rule():
    for m in (1, 16, 64, 65, 512):
        d, t = ql.qlinear_policy_lookup(4, m, 4096, 4096)
        assert not t and tune.rule_choice(m) == (d["strategy"], d["warps_per_unit"], d["ctas"])


def test_committed_b200_table_installs_and_covers_its_layers():
    import json
    with open(ql.default_policy_path()) as f:
        table = json.load(f)
    assert ql.load_policy() == len(table["entries"]) > 0
    layers = {(e["fmt"], e["K"], e["N"]) for e in table["entries"]}
    assert len(layers) == 24                       # 4 formats x 6 layers
    for fmt, K, N in layers:
        own = sorted((e["m_lo"], e["m_hi"]) for e in table["entries"]
                     if (e["fmt"], e["K"], e["N"]) == (fmt, K, N))
        assert own[0][0] == 1 and own[-1][1] == M_MAX
        assert all(b[0] == a[1] + 1 for a, b in zip(own, own[1:]))   # contiguous, disjoint
        for m in (1, 7, 16, 17, 64, 65, 4096):
            assert ql.qlinear_policy_lookup(fmt, m, N, K)[1]
    # the validation pairs were measured for every layer and M of the sweep
    assert len(table["validation"]) == 24 * len(table["M"])
