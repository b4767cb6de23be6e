"""Host-only checks of phase tracing: the normal library refuses to trace, the
traced build compiles and exports the same C ABI, and the trace summary turns
a table of (global ns, cycles) entries into the right per-kernel times."""
import ctypes

import numpy as np

import kv_cache_decode_csa2_b200 as K
from kv_cache_decode_csa2_b200 import build as Bd
from kv_cache_decode_csa2_b200 import csa2 as B
from kv_cache_decode_csa2_b200 import trace as T


def test_normal_build_does_not_trace():
    L = K.lib()
    assert L.csa2_trace_table_bytes() == T.KERNELS * T.CTAS * T.POINTS * 2 * 8
    assert L.csa2_trace_attach(None) == 2          # CSA2_ERR_UNSUPPORTED, nothing touched


def test_traced_build_exports_the_same_abi():
    path = Bd.build(trace=True)
    assert path != B.LIB_PATH
    L = ctypes.CDLL(path)                          # loaded beside the normal library, not instead of it
    for name in B.EXPORTS:
        assert hasattr(L, name), name


def _table():
    return np.zeros((T.KERNELS, T.CTAS, T.POINTS, 2), dtype=np.uint64)


def test_summary_times_from_a_known_table():
    t = _table()
    ghz = 2.0
    base = 10_000_000
    # kernel 5 (zero): one CTA, entry at base, done 1 us later
    t[5, 0, 0] = (base, 0)
    t[5, 0, 1] = (base + 1000, 2000)
    # kernel 0 (index score): two CTAs entering 2 us and 3 us after base;
    # point 1 after 0.5 us (CTA 0) and 1.5 us (CTA 1), point 9 after 20 us
    for c, (start, p1) in enumerate([(2000, 500), (3000, 1500)]):
        t[0, c, 0] = (base + start, 0)
        t[0, c, 1] = (base + start + p1, int(p1 * ghz))
        t[0, c, 9] = (base + start + 20000, int(20000 * ghz))
    stats = T.summarize(t, ghz)
    assert [s.name for s in stats] == ["zero", "index_score"]
    z, k1 = stats
    assert z.ctas == 1 and z.start_us == 0.0 and abs(z.end_us - 1.0) < 1e-9
    assert k1.ctas == 2 and abs(k1.start_us - 2.0) < 1e-9 and abs(k1.end_us - 23.0) < 1e-9
    names = [p.name for p in k1.points]
    assert names == ["entry", "prologue done", "exit"]
    entry, pro, ext = k1.points
    assert abs(entry.median_us - 2.5) < 1e-9 and abs(entry.max_us - 3.0) < 1e-9
    assert abs(pro.median_us - 3.5) < 1e-9 and abs(pro.max_us - 4.5) < 1e-9 and pro.reached == 2
    assert abs(ext.max_us - 23.0) < 1e-9
    text = T.format_report(stats, ghz)
    assert "index_score: 2 CTAs traced" in text and "prologue done" in text


def test_clock_rate_from_the_trace():
    t = _table()
    t[1, 3, 0] = (5_000_000, 0)
    t[1, 3, 8] = (5_010_000, 19_000)              # 10 us at 1.9 GHz
    t[1, 4, 0] = (5_000_000, 0)
    t[1, 4, 2] = (5_000_500, 900)                 # too short to measure: ignored
    assert abs(T.clock_ghz(t) - 1.9) < 1e-12
    assert T.clock_ghz(_table()) == 1.9           # nothing measurable: the default
    assert T.summarize(_table()) == []


def test_points_a_cta_did_not_reach_are_left_out():
    t = _table()
    t[3, 0, 0] = (1000, 0)
    t[3, 0, 8] = (3000, 4000)
    t[3, 1, 0] = (1500, 0)                        # this CTA recorded only its entry
    (s,) = T.summarize(t, 2.0)
    by = {p.name: p for p in s.points}
    assert by["entry"].reached == 2 and by["partial written"].reached == 1
    assert abs(by["partial written"].median_us - 2.0) < 1e-9
