"""End-to-end parity of flashloop_loop_step (loops 1..R) against the oracle
on the same seeded inputs.  Gate sets and selections must match exactly
(a selection may differ only inside a near-tie of the column mass); cached
codes may differ only where float rounding of the projection moved a value
across a rounding boundary; O and Y must be within relative L2 1e-2 per row."""
import numpy as np
import pytest
import torch

import oracle as O
from workload import CONFIGS, make_hidden_states, make_weights

pytestmark = pytest.mark.gpu

F = pytest.importorskip("cross_loop_sparse_b200.flashloop")
from gpu_helpers import bf16_rows, bf16_to_torch, row_rel_l2, torch_to_bf16_bits  # noqa: E402

TOL = 1e-2


def run_gpu(cfg, W, X, stream=None):
    p = F.Params.from_config(cfg)
    st = F.FlashLoopState(p)
    xs = [bf16_to_torch(x) for x in X]
    wqkv, wo = bf16_to_torch(W["wqkv"]), bf16_to_torch(W["wo"])
    snaps = {}
    for r in range(1, cfg.n_loops + 1):
        F.flashloop_loop_step(p, r, xs[r - 1], xs[r - 2] if r > 1 else None, wqkv, wo, st)
        torch.cuda.synchronize()
        snaps[r] = {
            "O": torch_to_bf16_bits(st["O"]),
            "Y": torch_to_bf16_bits(st["Y"]),
            "n": int(st["n_active"][r - 1].item()) if r > 1 else cfg.seq,
            "active": st[f"active{r}"].cpu().numpy().copy() if r > 1 else np.arange(cfg.seq),
        }
        if r >= 2:
            snaps[r]["cols"] = st.cols_for_loop(r).cpu().numpy().copy()
    assert st.error_code() == 0
    return p, st, snaps


def check_selection(gpu_cols, orc_cols, mass):
    """Equal sets, or different only between columns of (near-)equal mass."""
    g, o = set(gpu_cols.tolist()), set(np.asarray(orc_cols).tolist())
    if g == o:
        return 0
    only_g, only_o = sorted(g - o), sorted(o - g)
    band = 1e-5 * float(np.max(mass))
    kth = min(mass[list(o)])
    for j in only_g + only_o:
        assert abs(mass[j] - kth) <= band, (j, mass[j], kth)
    return len(only_g)


def compare(cfg, orc, snaps, heads, check_y):
    d, dh = cfg.d_model, cfg.head_dim
    cols = np.concatenate([np.arange(h * dh, (h + 1) * dh) for h in heads])
    worst = {}
    for r in range(1, cfg.n_loops + 1):
        s = snaps[r]
        act = orc.active[r]
        assert s["n"] == act.size
        assert np.array_equal(s["active"][: act.size], act)
        if r >= 2:
            for a, h in enumerate(heads):
                check_selection(s["cols"][h], orc.T[F.flashloop_selection_loop(F.Params.from_config(cfg), r)][a],
                                orc.colmass[1][a])
        og = bf16_rows(s["O"][act][:, cols])
        oo = bf16_rows(orc.O_hist[r][act])
        e = row_rel_l2(og, oo)
        worst[f"O{r}"] = float(e.max())
        assert e.max() < TOL, (r, e.max(), int(np.argmax(e)))
        if check_y:
            yg = bf16_rows(s["Y"][act])
            yo = bf16_rows(orc.Y_hist[r][act])
            ey = row_rel_l2(yg, yo)
            worst[f"Y{r}"] = float(ey.max())
            assert ey.max() < TOL, (r, ey.max())
    return worst


@pytest.mark.parametrize("name", ["tiny", "ouro14_4k"])
def test_loop_step_matches_oracle(name):
    cfg = CONFIGS[name]
    W = make_weights(cfg)
    X, _ = make_hidden_states(cfg)
    orc = O.OracleSequence(cfg, W, X).run()
    p, st, snaps = run_gpu(cfg, W, X)
    worst = compare(cfg, orc, snaps, list(range(cfg.n_heads)), True)
    print(name, worst)
    # cache codes: identical except where rounding of the projection moved a
    # value across a code boundary; reconstructions stay within the bound
    for name_, kv in (("k", orc.Kc), ("v", orc.Vc)):
        codes, s16 = kv.base
        got = st[f"{name_}_base"].cpu().numpy()
        assert np.mean(got != codes) < 1e-3
        assert np.max(np.abs(got.astype(int) - codes)) <= 1
        for r in range(2, cfg.n_loops + 1):
            n = orc.active[r].size
            gc = O.unpack_codes(st[f"{name_}_res{r}"][:n].cpu().numpy(), cfg.bits[r - 1])
            assert np.mean(gc != kv.res[r][0]) < 5e-3, (name_, r)


@pytest.mark.parametrize("name,heads", [("depth_8k_r8", [0, 9]), ("prefill_32k", [5])])
def test_loop_step_matches_oracle_on_held_heads(name, heads):
    cfg = CONFIGS[name]
    W = make_weights(cfg)
    X, _ = make_hidden_states(cfg)
    orc = O.OracleSequence(cfg, W, X, heads=heads).run()
    p, st, snaps = run_gpu(cfg, W, X)
    worst = compare(cfg, orc, snaps, heads, False)
    print(name, worst)
    # Y at full size: every row of the final Y is its final O times W_o^T
    # (float64 check on a sample of rows)
    rng = np.random.default_rng(0)
    wo = bf16_rows(W["wo"])
    rows = rng.choice(cfg.seq, size=64, replace=False)
    s = snaps[cfg.n_loops]
    want = bf16_rows(s["O"][rows]) @ wo.T
    assert row_rel_l2(bf16_rows(s["Y"][rows]), want).max() < TOL


def test_loop_steps_are_repeatable():
    """Loops 2..R re-run from the untouched loop-1 state give identical bytes."""
    cfg = CONFIGS["tiny"]
    W = make_weights(cfg)
    X, _ = make_hidden_states(cfg)
    p = F.Params.from_config(cfg)
    st = F.FlashLoopState(p)
    xs = [bf16_to_torch(x) for x in X]
    wqkv, wo = bf16_to_torch(W["wqkv"]), bf16_to_torch(W["wo"])
    F.flashloop_loop_step(p, 1, xs[0], None, wqkv, wo, st)
    outs = []
    for rep in range(2):
        for r in range(2, cfg.n_loops + 1):
            F.flashloop_loop_step(p, r, xs[r - 1], xs[r - 2], wqkv, wo, st)
        torch.cuda.synchronize()
        outs.append((torch_to_bf16_bits(st["O"]).copy(), torch_to_bf16_bits(st["Y"]).copy()))
    assert np.array_equal(outs[0][0], outs[1][0]) and np.array_equal(outs[0][1], outs[1][1])
