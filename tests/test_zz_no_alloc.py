"""flashloop_gate_noalloc, the gate entry point for callers that cannot
allocate device memory (a serving process with a frozen HBM budget, a host
framework that owns every allocation): it must give exactly what
flashloop_gate gives with a caller-provided workspace, call after call.

This file is collected last so that a stop-at-first-failure run has
already run every other test."""
import numpy as np
import pytest
import torch

import oracle as O
from workload import CONFIGS, make_hidden_states

pytestmark = pytest.mark.gpu

F = pytest.importorskip("cross_loop_sparse_b200.flashloop")


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _outputs(fn, p, x_cur, x_prev, prev, n_prev, S, extra):
    act = torch.full((S,), -7, dtype=torch.int32, device="cuda")
    slot = torch.full((S,), -7, dtype=torch.int32, device="cuda")
    n = torch.full((1,), -7, dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    fn(p, x_cur, x_prev, prev, n_prev, S, act, slot, n, S, *extra(err))
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    k = int(n.item())
    return k, act[:k].cpu().numpy(), slot.cpu().numpy()


@pytest.mark.parametrize("name", ["tiny", "ouro14_4k"])
def test_noalloc_gate_matches_workspace_gate_on_consecutive_calls(name):
    cfg = CONFIGS[name]
    X, _ = make_hidden_states(cfg)
    p = F.Params.from_config(cfg)
    S = cfg.seq
    xs = [_dev(x) for x in X]
    ws = torch.zeros(F.flashloop_workspace_bytes(p), dtype=torch.uint8, device="cuda")
    prev, n_prev = None, None
    cand = np.arange(S)
    for r in range(2, cfg.n_loops + 1):
        want = _outputs(F.flashloop_gate, p, xs[r - 1], xs[r - 2], prev, n_prev, S,
                        lambda err: (ws, err))
        # the workspace gate itself is the oracle's gate, bit for bit
        cand = O.gate(X[r - 1], X[r - 2], cand, cfg.tau)
        assert np.array_equal(want[1], cand), r
        for call in range(2):          # two calls in a row share the static scratch
            got = _outputs(F.flashloop_gate_noalloc, p, xs[r - 1], xs[r - 2], prev, n_prev, S,
                           lambda err: (err,))
            assert got[0] == want[0], (r, call)
            assert np.array_equal(got[1], want[1]), (r, call)
            assert np.array_equal(got[2], want[2]), (r, call)
        prev = torch.from_numpy(want[1].astype(np.int32)).cuda()
        n_prev = torch.tensor([want[0]], dtype=torch.int32, device="cuda")


def test_noalloc_gate_rejects_sizes_beyond_its_scratch():
    big = CONFIGS["tiny"]
    p = F.Params.from_config(big, seq=70000, capacity=[70000] * big.n_loops)
    x = torch.zeros((1, 8), dtype=torch.bfloat16, device="cuda")
    buf = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(F.FlashLoopError) as exc:
        F.flashloop_gate_noalloc(p, x, x, None, None, 70000, buf, buf, buf, 70000, buf)
    assert exc.value.status == -2
