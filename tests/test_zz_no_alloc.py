"""The allocation-free ranking entry point against the workspace one.

``da2_rank_noalloc`` serves callers that cannot allocate device memory when
they call in (a runtime that owns the whole GPU through its own arena, a plugin
hook inside another engine's execution path): its radix-select scratch is a
fixed array inside the library instead of a caller workspace.  Its results must
equal ``da2_rank_from_scores``'s exactly (integer outputs), on two calls in a
row with different scores, so that nothing left in the shared array by one
call leaks into the next.  This file is named to be collected last.
"""

import numpy as np
import pytest
import torch

from mixed_precision_block_b200.synth import Workload

pytestmark = pytest.mark.gpu


def _scores(nbh, nb, seed):
    rng = np.random.default_rng(seed)
    s = rng.random((nbh, nb, nb)).astype(np.float32)
    s[0] = rng.choice(np.array([0.0, 1e-3, 0.5], np.float32), size=(nb, nb))  # heavy ties
    s[1][rng.random((nb, nb)) < 0.4] = 0.0
    return torch.from_numpy(s).cuda()


def test_noalloc_rank_matches_workspace_rank_on_consecutive_calls():
    from mixed_precision_block_b200 import da2

    wl = Workload("noalloc", 2, 3, 3, 40, 24, 64, 0.5, (40.0, 20.0, 25.0, 15.0))
    p = da2.Problem.from_workload(wl)
    info = da2.da2_plan(p)
    nbh, nb = wl.B * wl.H, info.nb
    ws = da2.workspace(p)
    prec_map = torch.empty((nbh, nb, nb), dtype=torch.uint8, device="cuda")
    lists = torch.empty((nbh, nb, nb), dtype=torch.int16, device="cuda")
    counts = torch.empty((nbh, nb, 4), dtype=torch.int32, device="cuda")
    for call in range(2):
        s = _scores(nbh, nb, seed=10 + call)
        da2.da2_rank_from_scores(p, s, ws)
        da2.da2_rank_noalloc(p, s, prec_map, lists, counts)
        torch.cuda.synchronize()
        want_map = da2.view(p, ws, "MAP").cpu().numpy()
        want_counts = da2.view(p, ws, "COUNTS").cpu().numpy()
        want_lists = da2.view(p, ws, "LISTS").cpu().numpy()
        got_map, got_counts, got_lists = (t.cpu().numpy() for t in (prec_map, counts, lists))
        np.testing.assert_array_equal(got_map, want_map)
        np.testing.assert_array_equal(got_counts, want_counts)
        used = want_counts[..., :3].sum(-1)
        for bh in range(nbh):
            for qb in range(nb):
                n = used[bh, qb]
                np.testing.assert_array_equal(got_lists[bh, qb, :n], want_lists[bh, qb, :n])
        # the budget was handed out in full
        assert [(got_map[0] == x).sum() for x in (16, 8, 4)] == [info.n16, info.n8, info.n4]


def test_noalloc_rejects_more_heads_than_its_scratch_holds():
    from mixed_precision_block_b200 import da2

    wl = Workload("too_many", 1, da2.NOALLOC_MAX_HEADS + 1, 1, 8, 16, 64, 0.5, (50.0, 0.0, 0.0, 50.0))
    p = da2.Problem.from_workload(wl)
    nb = da2.da2_plan(p).nb
    s = torch.zeros((wl.H, nb, nb), dtype=torch.float32, device="cuda")
    m = torch.empty((wl.H, nb, nb), dtype=torch.uint8, device="cuda")
    lst = torch.empty((wl.H, nb, nb), dtype=torch.int16, device="cuda")
    c = torch.empty((wl.H, nb, 4), dtype=torch.int32, device="cuda")
    with pytest.raises(da2.Da2Error) as e:
        da2.da2_rank_noalloc(p, s, m, lst, c)
    assert e.value.code == da2.DA2_ERR_UNSUPPORTED
