"""Staged parity: each CUDA step runs on exactly the inputs the oracle's
step received (oracle -> GPU), and its outputs are compared with the
oracle's.  Integer work (gate, codes, top-k) must match bit for bit."""
import numpy as np
import pytest
import torch

import oracle as O
from workload import CONFIGS, make_hidden_states, make_weights

pytestmark = pytest.mark.gpu

F = pytest.importorskip("cross_loop_sparse_b200.flashloop")
from gpu_helpers import (bf16_rows, bf16_to_torch, f32, i32, row_rel_l2, torch_to_bf16_bits,  # noqa: E402
                         upload_cache, upload_cols, upload_q, upload_sets, upload_state_after)

_RUNS = {}


def oracle_run(name):
    if name not in _RUNS:
        cfg = CONFIGS[name]
        W = make_weights(cfg)
        X, planted = make_hidden_states(cfg)
        _RUNS[name] = (cfg, W, X, planted, O.OracleSequence(cfg, W, X).run())
    return _RUNS[name]


def new_state(cfg):
    p = F.Params.from_config(cfg)
    return p, F.FlashLoopState(p)


@pytest.mark.parametrize("name", ["tiny", "ouro14_4k"])
def test_gate_bit_exact(name):
    cfg, W, X, planted, orc = oracle_run(name)
    p, st = new_state(cfg)
    xs = [bf16_to_torch(x) for x in X]
    for r in range(2, cfg.n_loops + 1):
        D, P = O.gate_norms(X[r - 1], X[r - 2], orc.active[r - 1])
        rel = np.sqrt(D / P)
        assert np.min(np.abs(rel - cfg.tau)) > 1e-3 * cfg.tau   # no row sits on the threshold
        if r == 2:
            prev, nprev = None, None
        else:
            prev = i32(orc.active[r - 1])
            nprev = i32([orc.active[r - 1].size])
        act = torch.zeros(cfg.seq, dtype=torch.int32, device="cuda")
        slot = torch.full((cfg.seq,), 7, dtype=torch.int32, device="cuda")
        n = torch.zeros(1, dtype=torch.int32, device="cuda")
        F.flashloop_gate(p, xs[r - 1], xs[r - 2], prev, nprev, cfg.seq, act, slot, n, cfg.seq,
                         st["workspace"], st["err"])
        torch.cuda.synchronize()
        want = orc.active[r]
        assert int(n.item()) == want.size
        assert np.array_equal(act[: want.size].cpu().numpy(), want)
        ws = np.full(cfg.seq, -1, np.int32)
        ws[want] = np.arange(want.size)
        assert np.array_equal(slot.cpu().numpy(), ws)
    assert st.error_code() == 0


@pytest.mark.parametrize("name", ["tiny", "ouro14_4k"])
def test_kv_quant_chain_bit_exact_on_identical_inputs(name):
    cfg, W, X, planted, orc = oracle_run(name)
    p, st = new_state(cfg)
    k1 = f32(orc.k_exact[1].astype(np.float32).reshape(cfg.seq, -1))
    v1 = f32(orc.v_exact[1].astype(np.float32).reshape(cfg.seq, -1))
    F.flashloop_kv_quant_residual(p, 1, k1, v1, None, None, st)
    torch.cuda.synchronize()
    for name_, kv in (("k", orc.Kc), ("v", orc.Vc)):
        codes, s16 = kv.base
        assert np.array_equal(st[f"{name_}_base"].cpu().numpy(), codes)
        assert np.array_equal(st[f"{name_}_base_s"].cpu().numpy().view(np.uint16), s16.view(np.uint16))
    upload_sets(orc, st, cfg.n_loops)
    for r in range(2, cfg.n_loops + 1):
        act = orc.active[r]
        kr = f32(orc.k_exact[r].astype(np.float32).reshape(act.size, -1))
        vr = f32(orc.v_exact[r].astype(np.float32).reshape(act.size, -1))
        F.flashloop_kv_quant_residual(p, r, kr, vr, st[f"active{r}"], st["n_active"][r - 1:], st)
        torch.cuda.synchronize()
        for name_, kv in (("k", orc.Kc), ("v", orc.Vc)):
            codes, s16 = kv.res[r]
            packed = O.pack_codes(codes, cfg.bits[r - 1])
            got = st[f"{name_}_res{r}"][: act.size].cpu().numpy()
            assert np.array_equal(got, packed), (name_, r)
            gs = st[f"{name_}_res{r}_s"][: act.size].cpu().numpy().view(np.uint16)
            assert np.array_equal(gs, s16.view(np.uint16)), (name_, r)
    assert st.error_code() == 0


@pytest.mark.parametrize("name", ["tiny", "ouro14_4k"])
def test_topk_bit_exact_on_identical_mass(name):
    cfg, W, X, planted, orc = oracle_run(name)
    p, st = new_state(cfg)
    mass = f32(orc.colmass[1].astype(np.float32))
    out = torch.zeros((cfg.n_heads, cfg.k), dtype=torch.int32, device="cuda")
    F.flashloop_topk_columns(p, mass, None, 0, cfg.k, out)
    torch.cuda.synchronize()
    want = np.stack(orc.T[2])
    assert np.array_equal(out.cpu().numpy(), want)


def test_topk_ties_candidates_and_edges():
    cfg = CONFIGS["tiny"]
    p, st = new_state(cfg)
    rng = np.random.default_rng(4)
    H, S = cfg.n_heads, cfg.seq
    for trial in range(12):
        vals = rng.choice(np.array([0.0, -0.0, 1.5, 2.25, -3.0, 7.0], np.float32), size=(H, S))
        vals = np.where(rng.random((H, S)) < 0.3, rng.random((H, S)).astype(np.float32), vals)
        ncand = int(rng.integers(1, S + 1))
        cand = np.stack([np.sort(rng.choice(S, ncand, replace=False)) for _ in range(H)]).astype(np.int32)
        k = int(rng.integers(1, ncand + 1))
        out = torch.zeros((H, k), dtype=torch.int32, device="cuda")
        use_cand = trial % 3 != 0
        F.flashloop_topk_columns(p, f32(vals), i32(cand) if use_cand else None, ncand if use_cand else 0,
                                 k if use_cand else min(k, S), out)
        torch.cuda.synchronize()
        for h in range(H):
            cands = cand[h] if use_cand else np.arange(S)
            want = O.topk_columns(vals[h], cands, k if use_cand else min(k, S))
            assert np.array_equal(out[h].cpu().numpy(), want), (trial, h)
    # k = n: everything, ascending
    out = torch.zeros((H, S), dtype=torch.int32, device="cuda")
    F.flashloop_topk_columns(p, f32(np.zeros((H, S), np.float32)), None, 0, S, out)
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy(), np.tile(np.arange(S), (H, 1)))


def test_gate_bit_exact_at_32k():
    """The gate of loops 2..4 on the 32K workload's hidden states, each loop
    given the oracle's previous active set: sets, slot maps and counts
    bit-exact."""
    cfg = CONFIGS["prefill_32k"]
    X, _ = make_hidden_states(cfg)
    p = F.Params.from_config(cfg)
    st = F.FlashLoopState(p, kv_only=True)
    xs = [bf16_to_torch(x) for x in X]
    S = cfg.seq
    prev = np.arange(S)
    for r in range(2, cfg.n_loops + 1):
        want = O.gate(X[r - 1], X[r - 2], prev, cfg.tau)
        D, P = O.gate_norms(X[r - 1], X[r - 2], prev)
        assert np.min(np.abs(np.sqrt(D / P) - cfg.tau)) > 1e-3 * cfg.tau   # no row on the threshold
        act = torch.zeros(S, dtype=torch.int32, device="cuda")
        slot = torch.full((S,), 7, dtype=torch.int32, device="cuda")
        n = torch.zeros(1, dtype=torch.int32, device="cuda")
        F.flashloop_gate(p, xs[r - 1], xs[r - 2], None if r == 2 else i32(prev),
                         None if r == 2 else i32([prev.size]), S, act, slot, n, S, st["workspace"], st["err"])
        torch.cuda.synchronize()
        assert int(n.item()) == want.size, r
        assert np.array_equal(act[: want.size].cpu().numpy(), want), r
        ws = np.full(S, -1, np.int32)
        ws[want] = np.arange(want.size)
        assert np.array_equal(slot.cpu().numpy(), ws), r
        prev = want
    assert st.error_code() == 0


@pytest.mark.parametrize("with_candidates", [False, True])
def test_topk_bit_exact_at_32k_all_heads(with_candidates):
    """Top-k of S = 32768 columns on all 16 heads (one radix select over 32K
    keys per head), k = 3277: a column mass shaped like the workload's
    (about ln(S/j) with noise), exact ties planted at each head's k-th value
    and zeros of both signs; and the shrinking-budget form, k = 1638 among a
    head's 3277 previous columns.  Identical sets to the oracle's top-k."""
    cfg = CONFIGS["prefill_32k"]
    p = F.Params.from_config(cfg)
    H, S, k = cfg.n_heads, cfg.seq, cfg.k
    rng = np.random.default_rng(21)
    j = np.arange(S, dtype=np.float64)
    mass = (np.log(S / (j + 1.0))[None, :] * (1.0 + 0.05 * rng.standard_normal((H, S)))).astype(np.float32)
    for h in range(H):
        kth = np.sort(mass[h])[::-1][k - 1]
        mass[h, rng.choice(S, 40, replace=False)] = kth
        z = rng.choice(S, 20, replace=False)
        mass[h, z] = np.where(rng.random(20) < 0.5, np.float32(0.0), np.float32(-0.0))
    if with_candidates:
        cand = np.stack([O.topk_columns(mass[h], np.arange(S), k) for h in range(H)]).astype(np.int32)
        kk = (k + 1) // 2
        for h in range(H):   # ties at the new k-th value inside the candidates
            vals = mass[h, cand[h]]
            kth = np.sort(vals)[::-1][kk - 1]
            mass[h, cand[h][rng.choice(k, 12, replace=False)]] = kth
        want = np.stack([O.topk_columns(mass[h], cand[h], kk) for h in range(H)])
        out = torch.zeros((H, kk), dtype=torch.int32, device="cuda")
        F.flashloop_topk_columns(p, f32(mass), i32(cand), k, kk, out)
    else:
        want = np.stack([O.topk_columns(mass[h], np.arange(S), k) for h in range(H)])
        out = torch.zeros((H, k), dtype=torch.int32, device="cuda")
        F.flashloop_topk_columns(p, f32(mass), None, 0, k, out)
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy(), want)


@pytest.mark.parametrize("name", ["tiny", "ouro14_4k"])
def test_gathered_qkv_projection(name):
    cfg, W, X, planted, orc = oracle_run(name)
    p, st = new_state(cfg)
    wqkv = bf16_to_torch(W["wqkv"])
    d = cfg.d_model
    for r in (1, 2, cfg.n_loops):
        act = orc.active[r]
        n = act.size
        q = torch.zeros((cfg.seq, d), dtype=torch.bfloat16, device="cuda")
        k = torch.zeros((cfg.seq, d), dtype=torch.float32, device="cuda")
        v = torch.zeros_like(k)
        if r == 1:
            F.flashloop_qkv_gathered(p, bf16_to_torch(X[0]), None, None, cfg.seq, wqkv, st["rope_cs"], q, k, v)
        else:
            F.flashloop_qkv_gathered(p, bf16_to_torch(X[r - 1]), i32(act), i32([n]), cfg.seq, wqkv,
                                     st["rope_cs"], q, k, v)
        torch.cuda.synchronize()
        kk = k[:n].cpu().numpy().astype(np.float64)
        vv = v[:n].cpu().numpy().astype(np.float64)
        assert row_rel_l2(kk, orc.k_exact[r].reshape(n, d)).max() < 1e-5
        assert row_rel_l2(vv, orc.v_exact[r].reshape(n, d)).max() < 1e-5
        qg = bf16_rows(torch_to_bf16_bits(q[act]))
        qo = bf16_rows(orc.q[r][act].reshape(n, d))
        # bf16 storage of the same float32/float64 value: almost always the
        # same bits, and within a bf16 rounding step per row otherwise (an
        # element whose dot product nearly cancels can differ more in
        # relative terms, so the bound is taken per row)
        assert row_rel_l2(qg, qo).max() < 2.0 ** -8
        assert np.mean(qg == qo) > 0.99


@pytest.mark.parametrize("name", ["tiny", "ouro14_4k"])
def test_attention_update_staged(name):
    cfg, W, X, planted, orc = oracle_run(name)
    p, st = new_state(cfg)
    d, H, dh, S = cfg.d_model, cfg.n_heads, cfg.head_dim, cfg.seq
    upload_cache(orc, st, cfg.n_loops)
    upload_sets(orc, st, cfg.n_loops)
    # loop 1: dense attention and column mass
    upload_q(orc, st, 1)
    F.flashloop_selcol_dequant(p, 1, st)
    F.flashloop_sparse_attn_update(p, 1, st, 1)
    torch.cuda.synchronize()
    og = bf16_rows(torch_to_bf16_bits(st["O"]))
    oo = bf16_rows(orc.O_hist[1])
    assert row_rel_l2(og, oo).max() < 1e-2
    cm = st["colmass0"].cpu().numpy().astype(np.float64)
    assert np.max(np.abs(cm - orc.colmass[1]) / np.maximum(orc.colmass[1], 1e-3)) < 1e-2
    assert np.allclose(cm.sum(axis=1), S, rtol=1e-3)
    for r in range(2, cfg.n_loops + 1):
        upload_state_after(orc, st, r - 1)
        upload_q(orc, st, r - 1)
        upload_q(orc, st, r)
        upload_cols(orc, st, r)
        F.flashloop_selcol_dequant(p, r, st)
        F.flashloop_sparse_attn_update(p, r, st, 0)
        torch.cuda.synchronize()
        act = orc.active[r]
        og = bf16_rows(torch_to_bf16_bits(st["O"][act]))
        oo = bf16_rows(orc.O_hist[r][act])
        err = row_rel_l2(og, oo)
        assert err.max() < 1e-2, (r, err.max())
        m, Z, N = orc.hist[r]
        i = st.q_slot(r)
        Ng = st[f"N{i}"].cpu().numpy()[:, act].astype(np.float64)
        Zg = st[f"Z{i}"].cpu().numpy()[:, act].astype(np.float64)
        mg = st[f"m{i}"].cpu().numpy()[:, act].astype(np.float64)
        # the state is defined up to the common factor e^m: compare N e^m and Z e^m
        sc_g = np.exp(mg - m[:, act])
        assert np.max(np.abs(Zg * sc_g - Z[:, act]) / Z[:, act]) < 1e-3
        ref = np.linalg.norm(N[:, act], axis=-1)
        assert np.max(np.linalg.norm(Ng * sc_g[..., None] - N[:, act], axis=-1) / ref) < 1e-2
    assert st.error_code() == 0


@pytest.mark.parametrize("name", ["tiny", "ouro14_4k"])
def test_out_projection_staged(name):
    cfg, W, X, planted, orc = oracle_run(name)
    p, st = new_state(cfg)
    r = 2
    act = orc.active[r]
    o = bf16_to_torch(orc.O_hist[r])
    y = torch.zeros((cfg.seq, cfg.d_model), dtype=torch.bfloat16, device="cuda")
    F.flashloop_out_proj(p, o, i32(act), i32([act.size]), cfg.seq, bf16_to_torch(W["wo"]), y)
    torch.cuda.synchronize()
    yg = bf16_rows(torch_to_bf16_bits(y[act]))
    yo = O.out_projection(orc.O_hist[r][act], W["wo"])
    assert row_rel_l2(yg, bf16_rows(yo)).max() < 1e-2
    # rows outside the active set are untouched
    inactive = np.setdiff1d(np.arange(cfg.seq), act)
    assert torch.count_nonzero(y[inactive].float()).item() == 0


@pytest.mark.parametrize("name", ["tiny", "ouro14_4k"])
def test_fused_projection_quantiser_matches_unfused(name):
    """flashloop_qkv_quant (projection epilogue writes the codes) against
    flashloop_qkv_gathered + flashloop_kv_quant_residual on the same device
    inputs: identical q bits and identical cache bytes at every loop."""
    cfg, W, X, planted, orc = oracle_run(name)
    p, sa = new_state(cfg)
    _, sb = new_state(cfg)
    upload_sets(orc, sa, cfg.n_loops)
    upload_sets(orc, sb, cfg.n_loops)
    wqkv = bf16_to_torch(W["wqkv"])
    d, S = cfg.d_model, cfg.seq
    k = torch.zeros((S, d), dtype=torch.float32, device="cuda")
    v = torch.zeros_like(k)
    for r in range(1, cfg.n_loops + 1):
        x = bf16_to_torch(X[r - 1])
        qa = torch.zeros((S, d), dtype=torch.bfloat16, device="cuda")
        qb = torch.zeros_like(qa)
        if r == 1:
            F.flashloop_qkv_gathered(p, x, None, None, S, wqkv, sa["rope_cs"], qa, k, v)
            F.flashloop_kv_quant_residual(p, 1, k, v, None, None, sa)
            F.flashloop_qkv_quant(p, 1, x, None, None, wqkv, sb, qb)
        else:
            act, n = sa[f"active{r}"], sa["n_active"][r - 1:]
            F.flashloop_qkv_gathered(p, x, act, n, S, wqkv, sa["rope_cs"], qa, k, v)
            F.flashloop_kv_quant_residual(p, r, k, v, act, n, sa)
            F.flashloop_qkv_quant(p, r, x, sb[f"active{r}"], sb["n_active"][r - 1:], wqkv, sb, qb)
        torch.cuda.synchronize()
        assert torch.equal(qa.view(torch.int16), qb.view(torch.int16)), r
        keys = ["k_base", "k_base_s", "v_base", "v_base_s"] if r == 1 else \
            [f"k_res{r}", f"k_res{r}_s", f"v_res{r}", f"v_res{r}_s"]
        for key in keys:
            assert torch.equal(sa[key].view(torch.uint8), sb[key].view(torch.uint8)), (r, key)
    assert sa.error_code() == 0 and sb.error_code() == 0
