"""End-to-end parity of the sublayer (loops 1..R) against the oracle on the
same seeded inputs, in two forms.

Chained (the parity bar): every loop runs through the C-ABI calls that
flashloop_loop_step makes (gate, fused projection + quantiser, top-k,
selected-column rebuild, attention update, output projection).  After each
call that takes an integer decision the GPU's result is checked against the
oracle's (active sets exact; codes equal except where the float32
tensor-core projection and the float64 oracle projection fall on two sides
of a rounding boundary, and then by one step; selections equal except among
columns of near-equal mass), and the oracle's decision is written into the
GPU state before the chain goes on, so both sides attend over the same
cache bytes and columns.  Data flows oracle -> GPU only.  O and Y must then
be within relative L2 1e-2 on every active row of every loop.

Free-running: flashloop_loop_step alone.  The same integer checks hold; the
per-row O and Y errors are printed (a code that flipped at a rounding
boundary moves one INT2 step, so a row may move by about 1e-2)."""
import numpy as np
import pytest
import torch

import oracle as O
from workload import CONFIGS, make_hidden_states, make_weights

pytestmark = pytest.mark.gpu

F = pytest.importorskip("cross_loop_sparse_b200.flashloop")
from gpu_helpers import bf16_rows, bf16_to_torch, row_rel_l2, torch_to_bf16_bits  # noqa: E402

TOL = 1e-2


def run_gpu(cfg, W, X, stream=None, topk=None, token_budgets=None, fixed_mass=False, tau=None):
    p = F.Params.from_config(cfg, topk=topk, token_budgets=token_budgets, fixed_mass=fixed_mass, tau=tau)
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
    """Equal sets, or different only between columns of (near-)equal mass.
    Returns the columns that are in one set only."""
    g, o = set(gpu_cols.tolist()), set(np.asarray(orc_cols).tolist())
    if g == o:
        return set()
    only = (g - o) | (o - g)
    band = 1e-5 * float(np.max(mass))
    kth = min(mass[list(o)])
    for j in only:
        assert abs(mass[j] - kth) <= band, (j, mass[j], kth)
    return only


def gpu_reconstruct(st, cfg, name, tokens, loop, slots):
    """Khat/Vhat of the GPU cache (float64), rebuilt here from its bytes."""
    base = st[f"{name}_base"].cpu().numpy()[tokens].astype(np.float64)
    s = st[f"{name}_base_s"].cpu().numpy()[tokens].astype(np.float64)
    acc = base * np.repeat(s, 32, axis=-1)
    scale = np.repeat(s, 32, axis=-1)
    for l in range(2, loop + 1):
        sl = slots[l][tokens]
        have = sl >= 0
        if not have.any():
            continue
        c = O.unpack_codes(st[f"{name}_res{l}"].cpu().numpy()[sl[have]], cfg.bits[l - 1]).astype(np.float64)
        sc = np.repeat(st[f"{name}_res{l}_s"].cpu().numpy()[sl[have]].astype(np.float64), 32, axis=-1)
        acc[have] += c * sc
        if l == loop:
            scale[have] = sc
    return acc, scale


def check_caches(cfg, orc, st, heads):
    """Both caches quantise (almost) the same keys and values: wherever they
    differ the difference stays inside the two quantisers' rounding bounds."""
    slots = {r: orc.Kc.slot[r] for r in range(2, cfg.n_loops + 1)}
    hidx = np.array(heads)
    for r in range(1, cfg.n_loops + 1):
        toks = orc.active[r]
        for name, kv in (("k", orc.Kc), ("v", orc.Vc)):
            g, sg = gpu_reconstruct(st, cfg, name, toks, r, slots)
            g, sg = g[:, hidx], sg[:, hidx]
            o = kv.reconstruct(toks, r).astype(np.float64)
            so = np.repeat((kv.base[1] if r == 1 else kv.res[r][1]).astype(np.float64), 32, axis=-1)
            diff = np.abs(g - o)
            bound = (sg + so) / 2 * (1 + 1e-3) + 1e-4 * np.abs(o) + 1e-5
            assert np.all(diff <= bound), (name, r, float((diff - bound).max()))


def compare(cfg, orc, snaps, st, heads, check_y, topk=None):
    """Free-running run: active sets exact, selections exact up to near-ties,
    every cached reconstruction inside both quantisers' rounding bounds.
    Returns per loop the (median, worst) relative L2 of the O (and Y) rows,
    printed as a diagnostic."""
    dh = cfg.head_dim
    cols = held_cols(cfg, heads)
    check_caches(cfg, orc, st, heads)
    worst = {}
    sel_loop = {r: F.flashloop_selection_loop(F.Params.from_config(cfg, topk=topk), r)
                for r in range(2, cfg.n_loops + 1)}
    for r in range(1, cfg.n_loops + 1):
        s = snaps[r]
        act = orc.active[r]
        assert s["n"] == act.size
        assert np.array_equal(s["active"][: act.size], act)
        if r >= 2:
            for a, h in enumerate(heads):
                # the mass that loop's selection ranked: the dense loop-1 mass, or the
                # previous sparse loop's for a shrinking budget
                mass = orc.colmass[sel_loop[r] - 1][a]
                check_selection(s["cols"][h], orc.T[sel_loop[r]][a], mass)
        og = bf16_rows(s["O"][act][:, cols])
        oo = bf16_rows(orc.O_hist[r][act])
        e = row_rel_l2(og, oo)
        worst[f"O{r}"] = (round(float(np.median(e)), 5), round(float(e.max()), 5))
        if check_y:
            ey = row_rel_l2(bf16_rows(s["Y"][act]), bf16_rows(orc.Y_hist[r][act]))
            worst[f"Y{r}"] = (round(float(np.median(ey)), 5), round(float(ey.max()), 5))
    return worst


def held_cols(cfg, heads):
    dh = cfg.head_dim
    return np.concatenate([np.arange(h * dh, (h + 1) * dh) for h in heads])


def force_codes(cfg, orc, st, r, heads):
    """Loop r's codes and scales: the GPU's equal the oracle's except at rare
    rounding boundaries (and then by one step); the oracle's are then written
    over the held heads' part of the GPU streams."""
    for name, kv in (("k", orc.Kc), ("v", orc.Vc)):
        if r == 1:
            codes, s16 = kv.base
            got = st[f"{name}_base"].cpu().numpy()[:, heads]
            gs = st[f"{name}_base_s"].cpu().numpy()[:, heads]
            limit = 1e-3
        else:
            n = orc.active[r].size
            codes, s16 = kv.res[r]
            got = O.unpack_codes(st[f"{name}_res{r}"][:n].cpu().numpy(), cfg.bits[r - 1])[:, heads]
            gs = st[f"{name}_res{r}_s"][:n].cpu().numpy()[:, heads]
            limit = 2e-3
        assert np.mean(got != codes) < limit, (name, r, float(np.mean(got != codes)))
        assert np.max(np.abs(got.astype(np.int32) - codes), initial=0) <= 1, (name, r)
        # a group scale is fp16(max|rho| / qmax), rho the value (loop 1) or the
        # residual against the previous reconstruction.  The float32 tensor-core
        # and float64 oracle projections differ by ~1e-7 of the value, and a
        # residual is ~1/254 (after INT8) to ~1/3500 (after INT4 + INT2) of it,
        # so a residual scale may move by that difference plus its own fp16
        # rounding: one fp16 step plus 1e-5 of the group's largest value bounds
        # it (a wrong scale would be off by about the scale itself)
        x = (orc.k_exact if name == "k" else orc.v_exact)[r]
        gmax = np.abs(x).reshape(x.shape[:-1] + (x.shape[-1] // 32, 32)).max(axis=-1)
        ds = np.abs(gs.astype(np.float64) - s16.astype(np.float64))
        bound = np.spacing(s16).astype(np.float64) + 1e-5 * gmax
        assert np.all(ds <= bound), (name, r, float((ds - bound).max()))
        if r == 1:
            sb = gs.view(np.uint16) != s16.view(np.uint16)
            assert np.mean(sb) < 1e-2, (name, r, float(np.mean(sb)))
        if r == 1:
            st[f"{name}_base"][:, heads] = torch.from_numpy(codes.astype(np.int8)).cuda()
            st[f"{name}_base_s"][:, heads] = torch.from_numpy(s16).cuda()
        else:
            packed = O.pack_codes(codes, cfg.bits[r - 1])
            st[f"{name}_res{r}"][:n, heads] = torch.from_numpy(packed).cuda()
            st[f"{name}_res{r}_s"][:n, heads] = torch.from_numpy(s16).cuda()


def force_selection(p, orc, st, r, heads):
    """Loop r's selection (a selecting loop): the GPU's equals the oracle's up
    to near-ties of the ranked mass; the oracle's is then written over the
    held heads' rows."""
    got = st[f"cols{r}"].cpu().numpy()
    for a, h in enumerate(heads):
        check_selection(got[h], orc.T[r][a], orc.colmass[r - 1][a])
    st[f"cols{r}"][heads] = torch.from_numpy(np.stack(orc.T[r]).astype(np.int32)).cuda()


def run_chained(cfg, W, X, orc, heads, check_y, topk=None, fixed_mass=False, tau=None):
    """Loops 1..R through the calls flashloop_loop_step makes, the oracle's
    codes and selections written into the GPU state after each is checked
    (oracle -> GPU); then O of the held heads (and Y, with every head held)
    within TOL on every active row.  Returns the per-loop worst errors."""
    p = F.Params.from_config(cfg, topk=topk, fixed_mass=fixed_mass, tau=tau)
    st = F.FlashLoopState(p)
    xs = [bf16_to_torch(x) for x in X]
    wqkv, wo = bf16_to_torch(W["wqkv"]), bf16_to_torch(W["wo"])
    cols = held_cols(cfg, heads)
    R = cfg.n_loops
    worst = {}
    for r in range(1, R + 1):
        cap = p.capacity[r - 1]
        if r == 1:
            act_t = n_t = None
            F.flashloop_qkv_quant(p, 1, xs[0], None, None, wqkv, st, st["q0"])
        else:
            prev = None if r == 2 else st[f"active{r - 1}"]
            nprev = None if r == 2 else st["n_active"][r - 2:]
            act_t, n_t = st[f"active{r}"], st["n_active"][r - 1:]
            F.flashloop_gate(p, xs[r - 1], xs[r - 2], prev, nprev, p.capacity[r - 2], act_t, st[f"slot{r}"],
                             n_t, cap, st["workspace"], st["err"])
            F.flashloop_qkv_quant(p, r, xs[r - 1], act_t, n_t, wqkv, st, st[f"q{st.q_slot(r)}"])
        torch.cuda.synchronize()
        act = orc.active[r]
        if r >= 2:
            assert int(st["n_active"][r - 1].item()) == act.size
            assert np.array_equal(st[f"active{r}"][: act.size].cpu().numpy(), act)
        force_codes(cfg, orc, st, r, heads)
        if r >= 2 and F.flashloop_selection_loop(p, r) == r:
            k = p.topk[r - 1]
            if r == 2:
                F.flashloop_topk_columns(p, st["colmass0"], None, 0, k, st[f"cols{r}"])
            else:
                ps = F.flashloop_selection_loop(p, r - 1)
                F.flashloop_topk_columns(p, st["colmass1"], st[f"cols{ps}"], p.topk[ps - 1], k, st[f"cols{r}"])
            torch.cuda.synchronize()
            force_selection(p, orc, st, r, heads)
        want_cm = 1 if r == 1 else int(r < R and p.topk[r] < p.topk[r - 1])
        F.flashloop_selcol_dequant(p, r, st)
        F.flashloop_sparse_attn_update(p, r, st, want_cm)
        F.flashloop_out_proj(p, st["O"], act_t, n_t, cap, wo, st["Y"])
        torch.cuda.synchronize()
        og = bf16_rows(torch_to_bf16_bits(st["O"])[act][:, cols])
        e = row_rel_l2(og, bf16_rows(orc.O_hist[r][act]))
        worst[f"O{r}"] = round(float(e.max(initial=0.0)), 5)
        assert np.all(e < TOL), (r, float(e.max()), int(act[np.argmax(e)]))
        if check_y:
            ey = row_rel_l2(bf16_rows(torch_to_bf16_bits(st["Y"])[act]), bf16_rows(orc.Y_hist[r][act]))
            worst[f"Y{r}"] = round(float(ey.max(initial=0.0)), 5)
            assert np.all(ey < TOL), (r, float(ey.max()), int(act[np.argmax(ey)]))
    assert st.error_code() == 0
    return worst


@pytest.mark.parametrize("name", ["tiny", "ouro14_4k"])
def test_loop_step_matches_oracle(name):
    cfg = CONFIGS[name]
    W = make_weights(cfg)
    X, _ = make_hidden_states(cfg)
    orc = O.OracleSequence(cfg, W, X).run()
    heads = list(range(cfg.n_heads))
    chained = run_chained(cfg, W, X, orc, heads, True)
    p, st, snaps = run_gpu(cfg, W, X)
    free = compare(cfg, orc, snaps, st, heads, True)
    print(name, "chained", chained, "free-running", free)
    # codes differ only where float rounding of the projection moved a value
    # across a code boundary: rare, and one step for the base
    for name_, kv in (("k", orc.Kc), ("v", orc.Vc)):
        codes, s16 = kv.base
        got = st[f"{name_}_base"].cpu().numpy()
        assert np.mean(got != codes) < 1e-3
        assert np.max(np.abs(got.astype(int) - codes)) <= 1
        for r in range(2, cfg.n_loops + 1):
            n = orc.active[r].size
            gc = O.unpack_codes(st[f"{name_}_res{r}"][:n].cpu().numpy(), cfg.bits[r - 1])
            assert np.mean(gc != kv.res[r][0]) < 2e-3, (name_, r)


@pytest.mark.parametrize("name,heads", [("depth_8k_r8", [0, 9]), ("prefill_32k", [0, 5, 15])])
def test_loop_step_matches_oracle_on_held_heads(name, heads):
    cfg = CONFIGS[name]
    W = make_weights(cfg)
    X, _ = make_hidden_states(cfg)
    orc = O.OracleSequence(cfg, W, X, heads=heads).run()
    chained = run_chained(cfg, W, X, orc, heads, False)
    p, st, snaps = run_gpu(cfg, W, X)
    free = compare(cfg, orc, snaps, st, heads, False)
    print(name, "chained", chained, "free-running", free)
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


def test_loop_step_shrinking_budgets():
    """Nested selections with shrinking budgets (40, 26, 13 columns): loops 3
    and 4 rank the previous sparse loop's column mass over its selection."""
    cfg = CONFIGS["tiny"]
    topk = [cfg.seq, 40, 26, 13]
    W = make_weights(cfg)
    X, _ = make_hidden_states(cfg)
    orc = O.OracleSequence(cfg, W, X, topk=topk).run()
    chained = run_chained(cfg, W, X, orc, list(range(cfg.n_heads)), True, topk=topk)
    p, st, snaps = run_gpu(cfg, W, X, topk=topk)
    assert [F.flashloop_selection_loop(p, r) for r in (2, 3, 4)] == [2, 3, 4]
    for r in (3, 4):
        cols = snaps[r]["cols"]
        prev = snaps[r - 1]["cols"]
        for h in range(cfg.n_heads):
            assert set(cols[h].tolist()) <= set(prev[h].tolist())  # nested
            assert cols[h].size == topk[r - 1] and np.all(np.diff(cols[h]) > 0)
    free = compare(cfg, orc, snaps, st, list(range(cfg.n_heads)), True, topk=topk)
    print("shrinking", "chained", chained, "free-running", free)


@pytest.mark.parametrize("seq,k", [(300, 30), (131, 14), (64, 64)])
def test_loop_step_ragged_sizes(seq, k):
    """Sequence lengths and budgets that cut through the 128-row, 64-column
    and 256-column tiles of every kernel (and k = S at 64)."""
    cfg = CONFIGS["tiny"].with_(seq=seq)
    topk = [seq] + [k] * (cfg.n_loops - 1)
    W = make_weights(cfg)
    X, _ = make_hidden_states(cfg)
    orc = O.OracleSequence(cfg, W, X, topk=topk).run()
    heads = list(range(cfg.n_heads))
    chained = run_chained(cfg, W, X, orc, heads, True, topk=topk)
    p, st, snaps = run_gpu(cfg, W, X, topk=topk)
    free = compare(cfg, orc, snaps, st, heads, True, topk=topk)
    print(seq, k, "chained", chained, "free-running", free)


def test_full_budget_zero_threshold_is_dense_attention():
    """tau = 0 and k = S: every token active and every column selected, so
    loop r's output is dense causal attention with q^(r) over Khat^(r), Vhat^(r)
    (the identity the method is built on), here on the GPU against a dense
    float64 evaluation of the GPU's own caches and queries."""
    cfg = CONFIGS["tiny"].with_(seq=192, tau=0.0)
    S, H, dh = cfg.seq, cfg.n_heads, cfg.head_dim
    topk = [S] * cfg.n_loops
    W = make_weights(cfg)
    X, _ = make_hidden_states(cfg)
    p = F.Params.from_config(cfg, topk=topk, tau=0.0)
    st = F.FlashLoopState(p)
    xs = [bf16_to_torch(x) for x in X]
    wqkv, wo = bf16_to_torch(W["wqkv"]), bf16_to_torch(W["wo"])
    slots = {}
    for r in range(1, cfg.n_loops + 1):
        F.flashloop_loop_step(p, r, xs[r - 1], xs[r - 2] if r > 1 else None, wqkv, wo, st)
        torch.cuda.synchronize()
        if r >= 2:
            assert int(st["n_active"][r - 1].item()) == S
            slots[r] = st[f"slot{r}"].cpu().numpy()
        og = bf16_rows(torch_to_bf16_bits(st["O"])).reshape(S, H, dh)
        q = bf16_rows(torch_to_bf16_bits(st[f"q{st.q_slot(r)}"])).reshape(S, H, dh)
        toks = np.arange(S)
        Kh, _ = gpu_reconstruct(st, cfg, "k", toks, r, slots)
        Vh, _ = gpu_reconstruct(st, cfg, "v", toks, r, slots)
        for h in range(H):
            s = (q[:, h, :] @ Kh[:, h, :].T) / np.sqrt(dh)
            s = np.where(np.tril(np.ones((S, S), bool)), s, -np.inf)
            pmat = np.exp(s - s.max(axis=1, keepdims=True))
            ref = (pmat @ Vh[:, h, :]) / pmat.sum(axis=1, keepdims=True)
            err = row_rel_l2(og[:, h, :], ref)
            assert err.max() < 1e-2, (r, h, err.max())
    assert st.error_code() == 0


def test_empty_active_set():
    """A loop where no token changes enough: the gate keeps nothing and the
    kernels of that loop run on zero rows; O and Y keep the previous loop's
    rows and the next loop finds no candidates."""
    cfg = CONFIGS["tiny"].with_(seq=128, tau=10.0)
    W = make_weights(cfg)
    X, _ = make_hidden_states(cfg)
    p = F.Params.from_config(cfg, tau=10.0)
    st = F.FlashLoopState(p)
    xs = [bf16_to_torch(x) for x in X]
    wqkv, wo = bf16_to_torch(W["wqkv"]), bf16_to_torch(W["wo"])
    F.flashloop_loop_step(p, 1, xs[0], None, wqkv, wo, st)
    torch.cuda.synchronize()
    o1 = torch_to_bf16_bits(st["O"]).copy()
    y1 = torch_to_bf16_bits(st["Y"]).copy()
    for r in range(2, cfg.n_loops + 1):
        F.flashloop_loop_step(p, r, xs[r - 1], xs[r - 2], wqkv, wo, st)
        torch.cuda.synchronize()
        assert int(st["n_active"][r - 1].item()) == 0
        assert np.all(st[f"slot{r}"].cpu().numpy() == -1)
    assert np.array_equal(torch_to_bf16_bits(st["O"]), o1)
    assert np.array_equal(torch_to_bf16_bits(st["Y"]), y1)
    assert st.error_code() == 0


def test_attention_rejects_unaligned_output():
    """The attention update moves q, N and O rows in 32-byte accesses: an
    output tensor that does not start on 32 bytes is refused before any
    launch, and the state is left as it was."""
    cfg = CONFIGS["tiny"]
    W = make_weights(cfg)
    X, _ = make_hidden_states(cfg)
    p = F.Params.from_config(cfg)
    st = F.FlashLoopState(p)
    xs = [bf16_to_torch(x) for x in X]
    wqkv, wo = bf16_to_torch(W["wqkv"]), bf16_to_torch(W["wo"])
    F.flashloop_loop_step(p, 1, xs[0], None, wqkv, wo, st)
    torch.cuda.synchronize()
    o_before = torch_to_bf16_bits(st["O"]).copy()
    good = st.c.O
    st.c.O = good + 16
    try:
        with pytest.raises(F.FlashLoopError) as exc:
            F.flashloop_sparse_attn_update(p, 1, st, 0)
        assert exc.value.status == -1  # FLASHLOOP_ERR_INVALID_ARG
    finally:
        st.c.O = good
    torch.cuda.synchronize()
    assert np.array_equal(torch_to_bf16_bits(st["O"]), o_before)
    assert st.error_code() == 0


@pytest.mark.parametrize("case", ["tiny", "tiny_shrinking", "tiny_dense", "ouro_heads"])
def test_loop_step_fixed_mass_matches_oracle(case):
    """The fixed-mass form (selected columns keep their cached mass) against
    the oracle's explicit per-row distributions: the tiny workload, shrinking
    budgets (loops 3 and 4 rank the fixed-mass column mass), tau = 0 with
    k = S (every loop is then dense attention), and the 1.4B-like shape on
    two heads."""
    cfg = CONFIGS["ouro14_4k"].with_(seq=1024) if case == "ouro_heads" else CONFIGS["tiny"]
    topk, tau, heads = None, None, list(range(cfg.n_heads))
    if case == "tiny_shrinking":
        topk = [cfg.seq, 40, 26, 13]
    elif case == "tiny_dense":
        cfg = cfg.with_(seq=192, tau=0.0)
        topk, tau = [cfg.seq] * cfg.n_loops, 0.0
    elif case == "ouro_heads":
        heads = [0, 9]
    W = make_weights(cfg)
    X, _ = make_hidden_states(cfg)
    orc = O.OracleSequence(cfg, W, X, heads=heads, topk=topk, tau=tau, fixed_mass=True).run()
    all_heads = len(heads) == cfg.n_heads
    chained = run_chained(cfg, W, X, orc, heads, all_heads, topk=topk, fixed_mass=True, tau=tau)
    p, st, snaps = run_gpu(cfg, W, X, topk=topk, fixed_mass=True, tau=tau)
    assert p.fixed_mass == 1
    free = compare(cfg, orc, snaps, st, heads, all_heads, topk=topk)
    print(case, "chained", chained, "free-running", free)
    # the GPU's factor g reproduces the cached mass: for an active row of the last
    # loop, the selected columns' probabilities sum to the oracle's M_i
    R = cfg.n_loops
    slot = st.q_slot(R)
    G = st[f"G{slot}"].cpu().numpy()
    m = st[f"m{slot}"].cpu().numpy()
    Z = st[f"Z{slot}"].cpu().numpy()
    assert np.all(np.isfinite(G)) and np.all(G[:, orc.active[R]] >= 0)
    for a, h in enumerate(heads):
        T = orc.T[F.flashloop_selection_loop(p, R)][a]
        for i in orc.active[R][::17]:
            J = T[T <= i]
            if J.size == 0:
                continue
            want = orc.P[a, i, J].sum()
            q = bf16_rows(torch_to_bf16_bits(st[f"q{slot}"])[i:i + 1]).reshape(cfg.n_heads, -1)[h]
            Kj = orc.Kc.reconstruct(J, R)[:, a].astype(np.float64)
            s_new = Kj @ q / np.sqrt(cfg.head_dim)
            got = G[h, i] * np.exp(s_new - m[h, i]).sum() / Z[h, i]
            assert abs(got - want) <= 2e-2 * want + 1e-6, (h, int(i), got, want)
    assert st.error_code() == 0

