"""The C ABI library on the host: it loads, exports every declared entry point,
plans like the oracle counts, and rejects bad arguments before any launch.
No device work happens here (CPU only)."""

import ctypes
import os
import re

import pytest

import oracle
from oracle import geometry as OG
from mixed_precision_block_b200.synth import WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def da2():
    from mixed_precision_block_b200 import build
    build.build()
    from mixed_precision_block_b200 import da2 as mod
    return mod


def _declared():
    src = open(os.path.join(ROOT, "include", "da2.h")).read()
    return sorted(set(re.findall(r"^\s*(?:int|const char\*)\s+(da2_\w+)\s*\(", src, re.M)))


def test_every_declared_symbol_is_exported(da2):
    names = _declared()
    assert len(names) >= 8
    lib = ctypes.CDLL(da2._LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(da2.EXPORTS)


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_plan_matches_oracle_counts(da2, name):
    wl = WORKLOADS[name]
    info = da2.da2_plan(da2.Problem.from_workload(wl))
    op = oracle.CONFIGS[name]
    assert (info.n16, info.n8, info.n4, info.nskip) == OG.budget_counts(op)
    assert info.nb == op.nb and info.N == op.N and info.Np == 64 * op.nb
    assert info.pairs_per_head == op.nb ** 2
    assert info.ws_bytes > 0 and info.ws_bytes % 256 == 0


@pytest.mark.parametrize("field,value,code", [
    ("d", 96, 2), ("d", 0, 2), ("rh", 4, 2), ("B", 0, 1), ("T", -1, 1), ("lam", 1.5, 1), ("lam", -0.1, 1),
])
def test_plan_rejects(da2, field, value, code):
    p = da2.Problem.from_workload(WORKLOADS["tiny"])
    setattr(p, field, value)
    with pytest.raises(da2.Da2Error) as e:
        da2.da2_plan(p)
    assert e.value.code == code


@pytest.mark.parametrize("budget", [(0, 50, 50, 10), (10, 10, 10, 10), (-1, 0, 1, 100), (50, 30, 30, -10)])
def test_plan_rejects_budgets(da2, budget):
    with pytest.raises(da2.Da2Error) as e:
        da2.da2_plan(da2.Problem.from_workload(WORKLOADS["tiny"], budget=budget))
    assert e.value.code == da2.DA2_ERR_ARG


def test_budget_within_rounding_is_accepted(da2):
    info = da2.da2_plan(da2.Problem.from_workload(WORKLOADS["video4bit"]))  # sums to 99.9
    assert info.nskip == 3167683


def test_entry_points_check_workspace_and_pointers_before_launch(da2):
    p = da2.Problem.from_workload(WORKLOADS["tiny"])
    lib = da2._lib
    big = da2.da2_plan(p).ws_bytes
    fake = ctypes.c_void_p(1 << 40)  # never dereferenced: validation fails first
    assert lib.da2_prepare(ctypes.byref(p), fake, fake, fake, None, big, None) == da2.DA2_ERR_WORKSPACE
    assert lib.da2_prepare(ctypes.byref(p), fake, fake, fake, ctypes.c_void_p((1 << 40) + 8), big,
                           None) == da2.DA2_ERR_WORKSPACE
    assert lib.da2_prepare(ctypes.byref(p), fake, fake, fake, fake, big - 1, None) == da2.DA2_ERR_WORKSPACE
    assert lib.da2_prepare(ctypes.byref(p), ctypes.c_void_p((1 << 40) + 2), fake, fake, fake, big,
                           None) == da2.DA2_ERR_ARG
    assert lib.da2_draft_rank(ctypes.byref(p), None, big, None) == da2.DA2_ERR_WORKSPACE
    assert lib.da2_attention(ctypes.byref(p), fake, fake, fake, fake, big, None, None) == da2.DA2_ERR_ARG
    assert lib.da2_dense_attention(1, 1, 64, 96, fake, fake, fake, fake, None) == da2.DA2_ERR_UNSUPPORTED
    assert lib.da2_dense_attention(1, 1, 0, 64, fake, fake, fake, fake, None) == da2.DA2_ERR_ARG
    # one tensor-core kernel covers the dense path: shorter sequences than one
    # 64-token block are refused, not sent to another kernel
    assert lib.da2_dense_attention(1, 1, 63, 128, fake, fake, fake, fake, None) == da2.DA2_ERR_UNSUPPORTED
    assert lib.da2_attention_wait_test(ctypes.byref(p), fake, fake, fake, fake, big, fake, 0, 0,
                                       None) == da2.DA2_ERR_ARG  # a zero wait bound
    assert lib.da2_check_status(ctypes.byref(p), None, big, None) == da2.DA2_ERR_WORKSPACE
    assert lib.da2_check_status(ctypes.byref(p), fake, big - 1, None) == da2.DA2_ERR_WORKSPACE
    n = ctypes.c_int()
    assert lib.da2_attention_occupancy(96, 0, ctypes.byref(n)) == da2.DA2_ERR_ARG
    assert lib.da2_attention_occupancy(128, 0, None) == da2.DA2_ERR_ARG


def test_workspace_views_are_disjoint_and_inside(da2):
    p = da2.Problem.from_workload(WORKLOADS["mid"])
    size = da2.da2_plan(p).ws_bytes
    base = 1 << 40
    spans = []
    for i, name in enumerate(da2.VIEWS):
        ptr, nbytes = ctypes.c_void_p(), ctypes.c_size_t()
        assert da2._lib.da2_debug_view(ctypes.byref(p), ctypes.c_void_p(base), i, ctypes.byref(ptr),
                                       ctypes.byref(nbytes)) == 0
        assert ptr.value % 256 == 0 and ptr.value >= base and ptr.value + nbytes.value <= base + size
        spans.append((ptr.value, ptr.value + nbytes.value, name))
    spans.sort()
    for a, b in zip(spans, spans[1:]):
        assert a[1] <= b[0], (a, b)


def test_status_strings(da2):
    assert da2.da2_status_string(0) == "ok"
    assert "workspace" in da2.da2_status_string(3)
    assert da2.da2_status_string(99) == "unknown status"
    assert "bounded wait" in da2.da2_status_string(5)


def test_host_path_sizes_and_argument_checks(da2):
    # two sets of (Q, K, V, O chunk + chunk workspace) plus two status words
    # per chunk (the attention kernel's and the V preparation's); a chunk of G
    # heads is the same problem with B = 1, H = G
    for wl, Gs in ((WORKLOADS["mid"], (1, 5, 12, 40)), (WORKLOADS["mid"].with_(H=100), (1, 3))):
        p = da2.Problem.from_workload(wl)
        info = da2.da2_plan(p)
        for G in Gs:
            Gc = min(G, wl.B * wl.H)
            pc = da2.Problem.from_workload(wl, B=1, H=Gc)
            chunk = -(-info.N * wl.d * 2 * Gc // 256) * 256
            nchunks = -(-(wl.B * wl.H) // Gc)
            status = -(-nchunks * 8 // 256) * 256  # 100 chunks: 1024 bytes, not 512
            want = 2 * (4 * chunk + da2.da2_plan(pc).ws_bytes) + status
            assert da2.da2_host_bytes(p, G) == want
    with pytest.raises(da2.Da2Error) as e:
        da2.da2_host_bytes(p, 0)
    assert e.value.code == da2.DA2_ERR_ARG
    # a missing device buffer is refused before any CUDA call
    null = ctypes.c_void_p(None)
    host = ctypes.c_void_p(16)
    rc = da2._lib.da2_forward_host(ctypes.byref(p), host, host, host, host, null, 0, 4, null)
    assert rc == da2.DA2_ERR_WORKSPACE
    rc = da2._lib.da2_forward_host(ctypes.byref(p), null, host, host, host, null, 0, 4, null)
    assert rc == da2.DA2_ERR_ARG
