"""Decode (B sequences x one new token) on the GPU against the oracle's
OracleDecode, through the C ABI.

Staged: the oracle's own cache bytes, queries, selection and running state
are uploaded, so that each loop's attention is checked on identical inputs
(O within 1e-2 per row, probabilities to float rounding, the selection
exact up to near-ties).  End to end: the context caches come from the GPU's
KV path and the token's q/k/v from its projection, so cached codes may
differ where float rounding of a projection crossed a code boundary; the
gate sets must be identical, O and Y within 1e-2 per row."""
import math

import numpy as np
import pytest
import torch

import oracle as O
from workload import CONFIGS, make_decode_tokens, make_hidden_states, make_weights

pytestmark = pytest.mark.gpu

F = pytest.importorskip("cross_loop_sparse_b200.flashloop")
from gpu_helpers import bf16_rows, bf16_to_torch, row_rel_l2, torch_to_bf16_bits  # noqa: E402

TOL = 1e-2
LOG2E = 1.0 / math.log(2.0)


def decode_cfg(seq, batch, **kw):
    return CONFIGS["tiny"].with_(seq=seq, batch=batch, decode=True, **kw)


def inputs(cfg):
    W = make_weights(cfg)
    ctx = [make_hidden_states(cfg, b)[0] for b in range(cfg.batch)]
    tok = [make_decode_tokens(cfg, b) for b in range(cfg.batch)]
    return W, ctx, tok


def concat_loops(ctx, R):
    return [np.concatenate([c[r] for c in ctx], axis=0) for r in range(R)]


def stack_tokens(tok, R):
    return [np.stack([t[r] for t in tok], axis=0) for r in range(R)]


def context_sets(orcs, S, R):
    """The concatenated active list of each loop (rows b*S + j)."""
    return {r: np.concatenate([b * S + o.ctx_active[r] for b, o in enumerate(orcs)]) for r in range(2, R + 1)}


def upload_oracle_caches(cfg, orcs, ctx, ds):
    """The oracle's K/V bytes in the GPU layout: context rows b*S + j with
    residual rows at their place in the concatenated active list, the token
    of sequence b at row b of the token streams."""
    S, R = cfg.seq, cfg.n_loops
    sets = context_sets(orcs, S, R)
    counts = np.zeros(F.MAX_LOOPS, np.int32)
    counts[0] = cfg.batch * S
    for r in range(2, R + 1):
        act = sets[r]
        ctx[f"active{r}"][: act.size].copy_(torch.from_numpy(act.astype(np.int32)))
        slot = np.full(cfg.batch * S, -1, np.int32)
        slot[act] = np.arange(act.size)
        ctx[f"slot{r}"].copy_(torch.from_numpy(slot))
        counts[r - 1] = act.size
    ctx["n_active"].copy_(torch.from_numpy(counts))
    for name in ("k", "v"):
        base_c, base_s, tok_c, tok_s = [], [], [], []
        res = {r: ([], []) for r in range(2, R + 1)}
        tres = {r: ([], []) for r in range(2, R + 1)}
        for o in orcs:
            kv = o.Kc if name == "k" else o.Vc
            codes, s16 = kv.base
            base_c.append(codes[:S])
            base_s.append(s16[:S])
            tok_c.append(codes[S])
            tok_s.append(s16[S])
            for r in range(2, R + 1):
                c, s = kv.res[r]
                sl = kv.slot[r]
                rows = sl[o.ctx_active[r]]
                res[r][0].append(c[rows])
                res[r][1].append(s[rows])
                tres[r][0].append(c[sl[S]])
                tres[r][1].append(s[sl[S]])
        ctx[f"{name}_base"].copy_(torch.from_numpy(np.concatenate(base_c).astype(np.int8)))
        ctx[f"{name}_base_s"].copy_(torch.from_numpy(np.concatenate(base_s)))
        ds[f"{name}_base"].copy_(torch.from_numpy(np.stack(tok_c).astype(np.int8)))
        ds[f"{name}_base_s"].copy_(torch.from_numpy(np.stack(tok_s)))
        for r in range(2, R + 1):
            bits = cfg.bits[r - 1]
            packed = O.pack_codes(np.concatenate(res[r][0]), bits)
            n = packed.shape[0]
            ctx[f"{name}_res{r}"][:n].copy_(torch.from_numpy(packed))
            ctx[f"{name}_res{r}_s"][:n].copy_(torch.from_numpy(np.concatenate(res[r][1])))
            ds[f"{name}_res{r}"].copy_(torch.from_numpy(O.pack_codes(np.stack(tres[r][0]), bits)))
            ds[f"{name}_res{r}_s"].copy_(torch.from_numpy(np.stack(tres[r][1])))


def check_selection(gpu_cols, orc_cols, mass, band):
    """Equal sets, or different only between columns whose mass is within
    `band` of the k-th largest."""
    g, o = set(gpu_cols.tolist()), set(np.asarray(orc_cols).tolist())
    if g == o:
        return 0
    kth = min(mass[list(o)])
    for j in (g - o) | (o - g):
        assert abs(mass[j] - kth) <= band, (j, mass[j], kth, band)
    return len(g - o)


@pytest.mark.parametrize("seq,batch", [(200, 3), (77, 2)])
def test_decode_attention_staged(seq, batch):
    cfg = decode_cfg(seq, batch)
    W, ctx_x, tok = inputs(cfg)
    orcs = [O.OracleDecode(cfg, W, ctx_x[b], tok[b]).run() for b in range(batch)]
    p = F.Params.from_config(cfg)
    ctx = F.DecodeContext(p)
    ds = F.DecodeState(p)
    upload_oracle_caches(cfg, orcs, ctx, ds)
    H, dh, R, S = cfg.n_heads, cfg.head_dim, cfg.n_loops, cfg.seq
    for r in range(1, R + 1):
        i = ds.q_slot(r)
        ds[f"q{i}"].copy_(bf16_to_torch(np.stack([o.q[r].reshape(-1) for o in orcs])))
        if r >= 2:
            ip = ds.q_slot(r - 1)
            ds[f"q{ip}"].copy_(bf16_to_torch(np.stack([o.q[r - 1].reshape(-1) for o in orcs])))
            ds["cols"].copy_(torch.from_numpy(np.stack([np.stack(o.T) for o in orcs]).astype(np.int32)))
            m = np.stack([o.state[r - 1][0] for o in orcs]) * LOG2E
            ds[f"m{ip}"].copy_(torch.from_numpy(m.astype(np.float32)))
            ds[f"Z{ip}"].copy_(torch.from_numpy(np.stack([o.state[r - 1][1] for o in orcs]).astype(np.float32)))
            ds[f"N{ip}"].copy_(torch.from_numpy(np.stack([o.state[r - 1][2] for o in orcs]).astype(np.float32)))
        F.flashloop_decode_attn(p, r, ctx, ds)
        if r == 1:
            F.flashloop_decode_select(p, ds)
        torch.cuda.synchronize()
        og = bf16_rows(torch_to_bf16_bits(ds["O"]))
        oo = bf16_rows(np.stack([o.O[r] for o in orcs]))
        err = row_rel_l2(og.reshape(batch * H, dh), oo.reshape(batch * H, dh))
        assert err.max() < TOL, (r, err.max())
        # the running state, up to the common factor e^m
        mg = ds[f"m{i}"].cpu().numpy().astype(np.float64) / LOG2E
        zg = ds[f"Z{i}"].cpu().numpy().astype(np.float64)
        mo = np.stack([o.state[r][0] for o in orcs])
        zo = np.stack([o.state[r][1] for o in orcs])
        assert np.max(np.abs(zg * np.exp(mg - mo) - zo) / zo) < 1e-3, r
        if r == 1:
            pg = ds["probs"].cpu().numpy().astype(np.float64)
            po = np.stack([o.probs for o in orcs])
            assert np.max(np.abs(pg - po) / np.maximum(po, 1e-30)) < 1e-4
            assert np.allclose(pg.sum(axis=-1), 1.0, atol=1e-4)
            cols = ds["cols"].cpu().numpy()
            for b, o in enumerate(orcs):
                for h in range(H):
                    assert np.all(np.diff(cols[b, h]) > 0) and cols[b, h, -1] <= S
                    check_selection(cols[b, h], o.T[h], po[b, h], 1e-5 * po[b, h].max())
    assert ds.error_code() == 0


def gpu_recon(name, tensors, rows, loop, bits, slots):
    """Xhat of the given rows of a GPU cache (float64), rebuilt from its bytes;
    slots[l] maps a row to its loop-l residual row (-1: none)."""
    base = tensors[f"{name}_base"].cpu().numpy()[rows].astype(np.float64)
    s = tensors[f"{name}_base_s"].cpu().numpy()[rows].astype(np.float64)
    acc = base * np.repeat(s, 32, axis=-1)
    scale = np.repeat(s, 32, axis=-1)
    for l in range(2, loop + 1):
        sl = slots[l][rows]
        have = sl >= 0
        if not have.any():
            continue
        c = O.unpack_codes(tensors[f"{name}_res{l}"].cpu().numpy()[sl[have]], bits[l - 1]).astype(np.float64)
        sc = np.repeat(tensors[f"{name}_res{l}_s"].cpu().numpy()[sl[have]].astype(np.float64), 32, axis=-1)
        acc[have] += c * sc
        if l == loop:
            scale[have] = sc
    return acc, scale


def check_recon(g, sg, o, so):
    """Both caches quantise (almost) the same values: any difference stays
    inside the two quantisers' rounding bounds."""
    diff = np.abs(g - o)
    bound = (sg + so) / 2 * (1 + 1e-3) + 1e-4 * np.abs(o) + 1e-5
    assert np.all(diff <= bound), float((diff - bound).max())


def run_decode_gpu(cfg, W, ctx_x, tok):
    p = F.Params.from_config(cfg)
    R = cfg.n_loops
    ctx = F.DecodeContext(p)
    ds = F.DecodeState(p)
    wqkv, wo = bf16_to_torch(W["wqkv"]), bf16_to_torch(W["wo"])
    ctx.prepare([bf16_to_torch(x) for x in concat_loops(ctx_x, R)], wqkv)
    xt = [bf16_to_torch(x) for x in stack_tokens(tok, R)]
    snaps = {}
    for r in range(1, R + 1):
        F.flashloop_decode_step(p, r, xt[r - 1], wqkv, wo, ctx, ds)
        torch.cuda.synchronize()
        snaps[r] = {"O": torch_to_bf16_bits(ds["O"]), "Y": torch_to_bf16_bits(ds["Y"])}
        if r == 1:
            snaps[r]["probs"] = ds["probs"].cpu().numpy().astype(np.float64)
            snaps[r]["cols"] = ds["cols"].cpu().numpy().copy()
    assert ctx.error_code() == 0 and ds.error_code() == 0
    return p, ctx, ds, snaps


@pytest.mark.parametrize("seq,batch", [(256, 2), (131, 3)])
def test_decode_step_matches_oracle(seq, batch):
    cfg = decode_cfg(seq, batch)
    W, ctx_x, tok = inputs(cfg)
    orcs = [O.OracleDecode(cfg, W, ctx_x[b], tok[b]).run() for b in range(batch)]
    p, ctx, ds, snaps = run_decode_gpu(cfg, W, ctx_x, tok)
    H, dh, R, S = cfg.n_heads, cfg.head_dim, cfg.n_loops, cfg.seq
    # gate sets of the contexts: identical
    sets = context_sets(orcs, S, R)
    n = ctx["n_active"].cpu().numpy()
    for r in range(2, R + 1):
        assert n[r - 1] == sets[r].size
        assert np.array_equal(ctx[f"active{r}"][: sets[r].size].cpu().numpy(), sets[r])
    # caches: context and token, every loop
    cslots = {r: ctx[f"slot{r}"].cpu().numpy() for r in range(2, R + 1)}
    tslots = {r: np.arange(batch) for r in range(2, R + 1)}
    for r in range(1, R + 1):
        for name in ("k", "v"):
            for b, o in enumerate(orcs):
                kv = o.Kc if name == "k" else o.Vc
                toks = np.arange(S) if r == 1 else o.ctx_active[r]
                g, sg = gpu_recon(name, ctx.t, b * S + toks, r, cfg.bits, cslots)
                ov = kv.reconstruct(toks, r)
                so = np.repeat((kv.base[1][toks] if r == 1 else kv.res[r][1][kv.slot[r][toks]]).astype(np.float64),
                               32, axis=-1)
                check_recon(g, sg, ov, so)
                g, sg = gpu_recon(name, ds.t, np.array([b]), r, cfg.bits, tslots)
                ov = kv.reconstruct(np.array([S]), r)
                so = np.repeat((kv.base[1][[S]] if r == 1 else kv.res[r][1][kv.slot[r][[S]]]).astype(np.float64),
                               32, axis=-1)
                check_recon(g, sg, ov, so)
    # loop-1 probabilities and the selection
    pg = snaps[1]["probs"]
    po = np.stack([o.probs for o in orcs])
    assert np.allclose(pg.sum(axis=-1), 1.0, atol=1e-4)
    perr = np.abs(pg - po)
    assert perr.max() < 1e-3 * po.max()
    swaps = 0
    for b, o in enumerate(orcs):
        for h in range(H):
            swaps += check_selection(snaps[1]["cols"][b, h], o.T[h], po[b, h], 2 * perr[b, h].max() + 1e-7)
    assert swaps <= 2
    worst = {}
    wo = bf16_rows(W["wo"])
    for r in range(1, R + 1):
        og = bf16_rows(snaps[r]["O"])
        oo = bf16_rows(np.stack([o.O[r] for o in orcs]))
        e = row_rel_l2(og, oo)
        worst[r] = float(e.max())
        assert e.max() < TOL, (r, e)
        yg = bf16_rows(snaps[r]["Y"])
        yo = bf16_rows(np.stack([o.Y[r] for o in orcs]))
        assert row_rel_l2(yg, yo).max() < TOL, r
        # Y is O W_o^T of the GPU's own O (float64 check)
        assert row_rel_l2(yg, og @ wo.T).max() < 4e-3
    print(worst, "swaps", swaps)


def test_decode_full_size_sampled():
    """decode_32k: 8 sequences x 32768-token contexts through the GPU path;
    two sequences and one head checked against the oracle."""
    cfg = CONFIGS["decode_32k"]
    W, ctx_x, tok = inputs(cfg)
    p, ctx, ds, snaps = run_decode_gpu(cfg, W, ctx_x, tok)
    H, dh, R, S = cfg.n_heads, cfg.head_dim, cfg.n_loops, cfg.seq
    h = 3
    cols = slice(h * dh, (h + 1) * dh)
    for b in (0, 5):
        o = O.OracleDecode(cfg, W, ctx_x[b], tok[b], heads=[h]).run()
        pg = snaps[1]["probs"][b, h]
        perr = np.abs(pg - o.probs[0])
        assert perr.max() < 1e-3 * o.probs[0].max()
        check_selection(snaps[1]["cols"][b, h], o.T[0], o.probs[0], 2 * perr.max() + 1e-9)
        for r in range(1, R + 1):
            og = bf16_rows(snaps[r]["O"][b:b + 1, cols])
            oo = bf16_rows(o.O[r][None, :])
            assert row_rel_l2(og, oo).max() < TOL, (b, r)
    # every row: probabilities sum to one, the selection is ascending and in range
    assert np.allclose(snaps[1]["probs"].sum(axis=-1), 1.0, atol=1e-3)
    c = snaps[1]["cols"]
    assert np.all(np.diff(c, axis=-1) > 0) and c.min() >= 0 and c.max() <= S
