"""Top-k token retention (the gate variant that keeps a per-loop budget of the
most-changed tokens) on the GPU against the oracle's gate_topk, and the loop
step running with it end to end."""
import numpy as np
import pytest
import torch

import oracle as O
from workload import CONFIGS, bf16_bits_to_f32, f32_to_bf16_bits, make_hidden_states, make_weights

pytestmark = pytest.mark.gpu

F = pytest.importorskip("cross_loop_sparse_b200.flashloop")
from gpu_helpers import bf16_to_torch, i32  # noqa: E402
from test_gpu_end_to_end import compare, run_gpu  # noqa: E402


def gpu_gate_topk(cfg, xc, xp, prev, budget):
    """One call of flashloop_gate_topk; prev = None (all tokens) or an ascending list."""
    S = xc.shape[0]
    p = F.Params.from_config(cfg, seq=S)
    ws = torch.zeros(F.flashloop_kv_workspace_bytes(p), dtype=torch.uint8, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    act = torch.full((S,), -7, dtype=torch.int32, device="cuda")
    slot = torch.full((S,), -7, dtype=torch.int32, device="cuda")
    n = torch.zeros(1, dtype=torch.int32, device="cuda")
    if prev is None:
        pa, pn, pc = None, None, S
    else:
        pa = i32(np.concatenate([prev, np.full(S - prev.size, -9)]).astype(np.int32))
        pn, pc = i32([prev.size]), S
    F.flashloop_gate_topk(p, bf16_to_torch(xc), bf16_to_torch(xp), pa, pn, pc, budget, act, slot, n, S, ws, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    k = int(n.item())
    return act[:k].cpu().numpy(), slot.cpu().numpy(), k


def keys_of(xc, xp, cand):
    D, P = O.gate_norms(xc, xp, cand)
    with np.errstate(divide="ignore", invalid="ignore"):
        return np.where(P > 0, D / np.where(P > 0, P, 1), np.where(D > 0, np.inf, 0))


def check_same_up_to_ties(got, want, cand, key, rel=1e-5):
    g, w = set(got.tolist()), set(want.tolist())
    if g == w:
        return
    kth = key[np.isin(cand, want)].min()
    for t in g ^ w:
        kt = key[np.searchsorted(cand, t)]
        assert abs(kt - kth) <= rel * abs(kth), (t, kt, kth)


@pytest.mark.parametrize("name", ["tiny", "ouro14_4k"])
def test_gate_topk_planted_budgets(name):
    """With the planted budgets the GPU keeps exactly the planted sets."""
    cfg = CONFIGS[name]
    X, planted = make_hidden_states(cfg)
    prev = None
    for r in range(2, cfg.n_loops + 1):
        cand = np.arange(cfg.seq) if prev is None else prev
        got, slot, k = gpu_gate_topk(cfg, X[r - 1], X[r - 2], prev, cfg.n_active(r))
        want = O.gate_topk(X[r - 1], X[r - 2], cand, cfg.n_active(r))
        assert np.array_equal(got, want) and np.array_equal(got, planted[r - 1])
        exp_slot = np.full(cfg.seq, -1)
        exp_slot[got] = np.arange(k)
        assert np.array_equal(slot, exp_slot)
        prev = got


@pytest.mark.parametrize("fracs", [(0.5, 0.2, 0.08), (1.0, 0.3, 0.31)])
def test_gate_topk_other_budgets(fracs):
    """Budgets that cut inside the planted sets (the change ratios of planted
    rows differ by a few percent): equal sets up to near-ties; a budget above
    the candidate count keeps every candidate."""
    cfg = CONFIGS["ouro14_4k"]
    X, _ = make_hidden_states(cfg)
    prev = None
    for r, f in zip(range(2, cfg.n_loops + 1), fracs):
        cand = np.arange(cfg.seq) if prev is None else prev
        budget = int(round(f * cfg.seq))
        got, _, k = gpu_gate_topk(cfg, X[r - 1], X[r - 2], prev, budget)
        want = O.gate_topk(X[r - 1], X[r - 2], cand, budget)
        assert k == min(budget, cand.size)
        check_same_up_to_ties(got, want, cand, keys_of(X[r - 1], X[r - 2], cand))
        prev = want


def test_gate_topk_ties_and_zero_rows():
    """Duplicated rows have bit-identical changes: the lower token wins the
    tie; a zero previous row that changed is kept first, one that did not is
    dropped last."""
    cfg = CONFIGS["tiny"]
    rng = np.random.default_rng(5)
    S, d = 300, cfg.d_model
    xp = f32_to_bf16_bits(rng.standard_normal((S, d)).astype(np.float32))
    scale = np.exp(rng.uniform(-4, 0, size=(S, 1))).astype(np.float32)
    xc = f32_to_bf16_bits(bf16_bits_to_f32(xp) + rng.standard_normal((S, d)).astype(np.float32) * scale)
    for a, b in [(10, 200), (11, 12), (150, 3)]:
        xp[b], xc[b] = xp[a], xc[a]
    xp[77] = 0
    xc[77] = f32_to_bf16_bits(np.full(d, 0.5, np.float32))
    xp[78] = 0
    xc[78] = 0
    cand = np.arange(S)
    key = keys_of(xc, xp, cand)
    for budget in (1, 17, 150, 299, 300, 310):
        got, _, k = gpu_gate_topk(cfg.with_(seq=S), xc, xp, None, min(budget, S))
        want = O.gate_topk(xc, xp, cand, min(budget, S))
        check_same_up_to_ties(got, want, cand, key)
        assert 77 in got
        if budget < S:
            assert 78 not in got
        for a, b in [(10, 200), (11, 12), (150, 3)]:
            lo, hi = min(a, b), max(a, b)
            if hi in got:
                assert lo in got  # the tie goes to the lower token


def test_loop_step_with_token_retention():
    """flashloop_loop_step with the top-k gate (budgets = the planted sizes)
    matches the oracle run with the same gate, end to end."""
    cfg = CONFIGS["tiny"]
    budgets = [cfg.seq] + [cfg.n_active(r) for r in range(2, cfg.n_loops + 1)]
    W = make_weights(cfg)
    X, planted = make_hidden_states(cfg)
    orc = O.OracleSequence(cfg, W, X, token_budgets=budgets).run()
    p, st, snaps = run_gpu(cfg, W, X, token_budgets=budgets)
    assert p.gate_topk == 1
    for r in range(2, cfg.n_loops + 1):
        assert np.array_equal(snaps[r]["active"][: snaps[r]["n"]], orc.active[r])
        assert np.array_equal(orc.active[r], planted[r - 1])
    worst = compare(cfg, orc, snaps, st, list(range(cfg.n_heads)), True)
    print(worst)
